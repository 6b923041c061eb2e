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
// The GEMM runs on CTA pairs (clusters of two, one per SM pair): an output
// tile is 256 tokens x 256 features, one tcgen05.mma.cta_group::2 per 16
// channels (M = 256, N = 256), both operands K-major from 128-byte-swizzled
// TMA tiles. CTA r of the pair loads its own 128 token rows of X and the
// r-th 128 of the tile's 256 rows of W, so each SM brings in 32 KB per 64
// channels for 2 x 128 x 256 x 64 multiply-adds (a single-CTA 128 x 256 tile
// needs 48 KB for half of that). Each CTA's tensor memory holds its 128
// tokens x 256 features; two accumulators alternate, so the epilogue of one
// tile overlaps the main loop of the next.
//
// A column tile is either 256 query features, written to Q, or the 128 key
// and 128 value features of a group of four heads. For a key/value tile the
// epilogue rounds k and v to bf16, applies ReLU (and RoPE) to k, sums ReLU(k)
// over the tokens (warp transpose-sums), stages phi(k) and v in shared memory
// and accumulates the four heads' phi(K)^T V with warp-level mma.sync
// (bf16 operands read with ldmatrix, fp32 accumulators in registers; every
// warp 16 rows of one head's 32 x 32 state, tokens in a fixed order), over
// the pair's consecutive tiles of the same head group (a "run"). At the end
// of a run each CTA writes its partial (S, z) to a slot of the workspace; a
// second kernel sums every head's slots in a fixed order, so S and z are
// bitwise reproducible.
//
// Tile order: token tiles are cut into chunks of L tiles; a run is one column
// tile over the token tiles of one chunk, and pair c takes runs c, c + pairs,
// c + 2 pairs, ... (L is chosen on the host so that the busiest pair's tile
// count stays within 3% of the best). All pairs then stand at about the same
// token tile of neighbouring chunks, so X comes from HBM about once and W
// stays in L2.
//
// Warp roles (320 threads per CTA): warps 0-7 epilogue (warp w reads TMEM
// lanes 32 (w % 4) .. + 31, i.e. token rows; warps 0-3 the first 128
// columns, 4-7 the last 128), warp 8 TMA producer (both CTAs), warp 9 TMEM
// allocation and, in the pair's first CTA, the MMA issuer (one thread).
// Every wait is bounded; a wait that gives up raises the CTA's abort flag and
// the device error word, and the CTA drains its copies and MMAs before it
// frees tensor memory. The pair meets at cluster barriers after set-up and
// before exit, so neither CTA leaves while the other may still touch its
// shared memory. No load is multicast.
#include <algorithm>

#include "la_tc_common.cuh"

namespace la {

// Device error word of this kernel: bit 0 = a bounded wait gave up.
__device__ unsigned g_qkv_error;

namespace {

using namespace sm100;

constexpr int kQkvEpiWarps = 8;
constexpr int kEpiThreads = kQkvEpiWarps * 32;        // 256
constexpr int kQkvThreads = kEpiThreads + 64;         // + TMA warp + MMA warp
constexpr int kWarpTma = 8;
constexpr int kWarpMma = 9;
constexpr int kTokCta = 128;               // tokens per CTA per tile (TMEM lanes)
constexpr int kTokPair = 2 * kTokCta;      // tokens per tile (MMA M, across the pair)
constexpr int kCols = 256;                 // output features per tile (MMA N)
constexpr int kKBlk = 64;                  // channels per stage
// TMA stages (6 stages, with the state staging cut into two rounds to make
// room, measured the same: the loop is not short of loads in flight).
constexpr int kQStages = 5;
constexpr int kBoxBytes = 128 * 128;       // [128 rows][64 bf16], 128-byte swizzle
constexpr int kQStageBytes = 2 * kBoxBytes;  // this CTA's X rows + its 128 rows of W
constexpr int kStgRow = 256;               // staging row: 128 bf16 features of a token
constexpr int kStgHalf = kTokCta * kStgRow;  // phi(K) or V of the CTA's 128 tokens
constexpr int kAccCols = 256;
constexpr int kQkvTmemCols = 2 * kAccCols;
constexpr int kBarEpi = 1;                 // named barrier of the epilogue warps
// One partial slot (per CTA of a pair): the state of 4 heads (4 x 32 x 32),
// then the key sums of every TMEM lane quadrant ([4 quadrants][4 heads][32]).
constexpr int kPartS = 4 * kD * kD;
constexpr int kPartFloats = kPartS + 4 * 4 * kD;

struct QSmem {  // byte offsets from the 1024-aligned base
  static constexpr int stages = 0;
  static constexpr int stg = stages + kQStages * kQStageBytes;
  static constexpr int bars = stg + 2 * kStgHalf;
  // full[S] empty[S] acc_full[2] acc_empty[2] mma_done
  static constexpr int nbars = 2 * kQStages + 5;
  static constexpr int misc = bars + nbars * 8;  // tmem base, abort flag
  static constexpr int bytes = misc + 16;
};
constexpr int kQSmemBytes = QSmem::bytes + 1024;
static_assert(kQSmemBytes <= 232448, "dynamic shared memory of one CTA");

// The static schedule, a function of (B, N, H, C) only. "Units" are CTA
// pairs; a tile is 256 tokens of one batch element x one column tile.
struct QkvSched {
  int B, N, H, C, HD;
  int NT;     // token tiles (of 256) per batch element
  int G;      // head groups of 4 (key/value column tiles)
  int QC;     // query column tiles of 256
  int CT;     // column tiles: G key/value, then QC query
  int KB;     // K-blocks of 64 channels
  int L;      // token tiles per chunk
  int NK;     // chunks per batch element
  int total;  // tiles
  int units;  // runs: B * NK * CT
  int pairs;  // CTA pairs; pair c takes runs c, c + pairs, c + 2 pairs, ...
};

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
  int first;  // kv: first tile of its run in this pair
  int last;   // kv: last tile of its run in this pair
};

// Run u (a column tile over the consecutive token tiles of one chunk): its
// first tile and the end of its tiles.
__host__ __device__ inline void run_span(const QkvSched& s, int u, int& i0, int& i1) {
  const int b = u / (s.NK * s.CT);
  const int rem = u - b * s.NK * s.CT;
  const int k = rem / s.CT, ct = rem - k * s.CT;
  const int len = chunk_len(s, k);
  i0 = chunk_begin(s, b, k) + ct * len;
  i1 = i0 + len;
}

// The tiles of one pair in order: its runs u = pair, pair + pairs, ...; at any
// moment all pairs stand at about the same token tile of neighbouring chunks,
// so each X tile is read from HBM about once and its other reads hit L2.
struct PairTiles {
  int u, i, beg, end, tl;  // run, tile, run's first tile and end, tiles done
  __device__ PairTiles(const QkvSched& s, int pair) : u(pair), i(0), beg(0), end(0), tl(0) {
    if (u < s.units) run_span(s, u, beg, end);
    i = beg;
  }
  __device__ bool valid(const QkvSched& s) const { return u < s.units; }
  __device__ void next(const QkvSched& s) {
    ++tl;
    if (++i == end) {
      u += s.pairs;
      if (u < s.units) run_span(s, u, beg, end);
      i = beg;
    }
  }
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

// Byte offset of 16-byte chunk c (0..15) of token row r in a staging half:
// rows of 256 bytes, chunks XOR-swizzled by the row so that 8 consecutive
// rows writing the same chunk hit 8 different bank groups.
__device__ __forceinline__ uint32_t stg_offset(int r, int c) {
  return static_cast<uint32_t>(r * kStgRow + ((c ^ (r & 15)) << 4));
}

// Four 8x8 bf16 matrices from shared memory, each transposed on the way
// (thread i gives the address of row i % 8 of matrix i / 8).
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                              uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// d (16 x 8, fp32) += a (16 x 16, bf16) * b (16 x 8, bf16): a warp-wide MMA
// for the small state product of the epilogue.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// cos and sin of pos * inv_freq for the key feature map: the angle is formed
// and reduced to [-pi, pi] in double (exact enough for any position), then
// evaluated with the hardware approximations, whose absolute error on
// [-pi, pi] (about 2^-21) is far below the bf16 rounding of phi(k) that
// follows.
__device__ __forceinline__ void rope_cs_fast(int pos, double inv_freq, float& c, float& s) {
  const double kTwoPi = 6.283185307179586476925286766559;
  const double a = static_cast<double>(pos) * inv_freq;
  const float r = static_cast<float>(a - kTwoPi * rint(a * (1.0 / kTwoPi)));
  __sincosf(r, &s, &c);
}

// ---------------------------------------------------------- CTA-pair PTX

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// All threads of both CTAs of the cluster.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::
          : "memory");
}

// Shared-memory address, in the cluster window, of the variable at the same
// offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

// 3D tiled load into this CTA's shared memory whose completion is counted on
// an mbarrier of either CTA of the pair (no multicast).
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* m,
                                                 uint32_t bar_cluster, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// TMEM allocation shared by the pair: the same warp of both CTAs, the same
// destination offset.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// D[tmem of both CTAs] (+)= A[smem, 128 rows per CTA] * B[smem, 128 of N per
// CTA]; bf16 inputs, fp32 accumulation; issued by one thread of CTA 0.
__device__ __forceinline__ void mma_pair_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on the mbarrier at this offset in both CTAs of the pair when
// the pair MMAs this thread issued so far have completed.
__device__ __forceinline__ void mma_pair_commit_both(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(static_cast<uint16_t>(3))
      : "memory");
}
// ... on this CTA's mbarrier only.
__device__ __forceinline__ void mma_pair_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

template <int kRope>
__global__ void __launch_bounds__(kQkvThreads, 1)
qkv_state_tc(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
             const QkvSched sc, const Rope rope, const __nv_bfloat16* __restrict__ bias,
             __nv_bfloat16* __restrict__ Q, float* __restrict__ part) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + QSmem::bars);  // CTA 0's count both
  uint64_t* empty = full + kQStages;
  uint64_t* acc_full = empty + kQStages;  // [2]
  uint64_t* acc_empty = acc_full + 2;     // [2], CTA 0's count both CTAs' epilogues
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + QSmem::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + QSmem::misc + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();
  const int pair = blockIdx.x >> 1;

  if (tid == 0) {
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * kQkvEpiWarps);  // one arrival per epilogue warp of the pair
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpTma && lane == 0) {
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_w);
  }
  cluster_sync_all();  // both CTAs' barriers are initialised before any remote use
  if (warp == kWarpMma) {
    tmem_alloc_pair(tmem_slot, kQkvTmemCols);
    tmem_relinquish_pair();
    tc_fence_before();
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
      for (PairTiles it(sc, pair); ok && it.valid(sc); it.next(sc)) {
        const Tile t = decode(sc, it.i, it.beg, it.end);
        const int y = t.nt * kTokPair + static_cast<int>(rank) * kTokCta;
        // this CTA's 128 rows of the tile's 256 rows of W: the group's keys
        // (CTA 0) or values (CTA 1), or half of 256 query rows. Rows past
        // H*32 of a section read as zero, as do tokens past N and channels
        // past C.
        const int wy = t.kv ? t.col * 128 : t.col * kCols + static_cast<int>(rank) * 128;
        const int wz = t.kv ? 1 + static_cast<int>(rank) : 0;
        for (int kb = 0; kb < sc.KB; ++kb, ++pos) {
          const int s = pos % kQStages;
          if (!(ok = mbar_wait(&empty[s], ((pos / kQStages) & 1) ^ 1, abort_flag, &g_qkv_error,
                               kErrWait)))
            break;
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * kQStageBytes);
          const uint32_t bar = map_rank(smem_u32(&full[s]), 0);
          uint8_t* st = smem + QSmem::stages + s * kQStageBytes;
          const int x = kb * kKBlk;
          tma_load_3d_pair(st, &tm_x, bar, x, y, t.b);
          tma_load_3d_pair(st + kBoxBytes, &tm_w, bar, x, wy, wz);
        }
      }
      // every load issued must have landed before the CTA frees its memory:
      // CTA 0's full barriers count both CTAs' bytes; CTA 1's loads have
      // landed once CTA 0's MMAs released the stages
      for (int qq = max(0, pos - kQStages); qq < pos; ++qq) {
        if (rank == 0)
          mbar_drain(&full[qq % kQStages], (qq / kQStages) & 1, &g_qkv_error, kErrWait);
        else
          mbar_drain(&empty[qq % kQStages], (qq / kQStages) & 1, &g_qkv_error, kErrWait);
      }
    }
  } else if (warp == kWarpMma) {
    // ----------------------------------------------------- MMA (CTA 0 only)
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = idesc_bf16_f32(kTokPair, kCols, 0, 0);
      int pos = 0;
      bool ok = true;
      for (PairTiles it(sc, pair); ok && it.valid(sc); it.next(sc)) {
        const int tl = it.tl, buf = tl & 1;
        // both CTAs' epilogues have read this accumulator's previous tile
        if (!(ok = mbar_wait(&acc_empty[buf], ((tl >> 1) & 1) ^ 1, abort_flag, &g_qkv_error,
                             kErrWait)))
          break;
        tc_fence_after();
        const uint32_t acc = tmem + buf * kAccCols;
        for (int kb = 0; kb < sc.KB; ++kb, ++pos) {
          const int s = pos % kQStages;
          if (!(ok = mbar_wait(&full[s], (pos / kQStages) & 1, abort_flag, &g_qkv_error,
                               kErrWait)))
            break;
          tc_fence_after();
          const uint32_t st = sbase + QSmem::stages + s * kQStageBytes;
          const uint64_t a0 = smem_desc_sw128(st, 16, 1024);
          const uint64_t b0 = smem_desc_sw128(st + kBoxBytes, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < kKBlk / 16; ++kk) {
            const uint64_t ad = desc_at(a0, kk * 32);
            const uint64_t bd = desc_at(b0, kk * 32);
            mma_pair_bf16(acc, ad, bd, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          mma_pair_commit_both(&empty[s]);  // both CTAs' stages are free again
        }
        if (!ok) break;
        mma_pair_commit_both(&acc_full[buf]);
      }
      mma_pair_commit(mma_done);
      mbar_drain(mma_done, 0, &g_qkv_error, kErrWait);
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int quad = warp & 3;       // TMEM lane quadrant: token rows 32 quad ..
    const int hf = warp >> 2;        // 0: columns 0-127 (keys), 1: 128-255 (values)
    const int row = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t stg = sbase + QSmem::stg + (hf ? kStgHalf : 0);
    const uint32_t stg_k = sbase + QSmem::stg, stg_v = stg_k + kStgHalf;
    // the state block this warp accumulates: head sh, rows 16 smb .. + 15,
    // all 32 columns (four 16 x 8 MMA accumulators); g, t4: the lane's place
    // in an accumulator fragment
    const int sh = warp >> 1, smb = warp & 1;
    const int g = lane >> 2, t4 = lane & 3;
    float sacc[4][4] = {};
    float zacc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    const uint32_t acc_empty_0[2] = {map_rank(smem_u32(&acc_empty[0]), 0),
                                     map_rank(smem_u32(&acc_empty[1]), 0)};
    for (PairTiles it(sc, pair); it.valid(sc); it.next(sc)) {
      const Tile t = decode(sc, it.i, it.beg, it.end);
      const int tl = it.tl, buf = tl & 1;
      const int n = t.nt * kTokPair + static_cast<int>(rank) * kTokCta + row;
      const bool valid = n < sc.N;
      // first feature (row of W, entry of the bias) of this warp's 128 columns
      const int f0 = t.kv ? (1 + hf) * sc.HD + t.col * 128 : t.col * kCols + hf * 128;
      const int f_end = t.kv ? (2 + hf) * sc.HD : sc.HD;
      // the bias of chunk ch (32 features as 16 bf16 pairs), loaded two chunks
      // ahead; the first two before the accumulator wait, so that their
      // latency hides behind it
      uint4 bq[2][4];
      auto load_bias = [&](int ch, uint4(&dst)[4]) {
        const int f = f0 + ch * 32;
        const bool have = bias != nullptr && f < f_end;
        const uint4* bp = reinterpret_cast<const uint4*>(bias + (have ? f : 0));
#pragma unroll
        for (int k = 0; k < 4; ++k) dst[k] = have ? __ldg(bp + k) : make_uint4(0u, 0u, 0u, 0u);
      };
      load_bias(0, bq[0]);
      load_bias(1, bq[1]);
      // RoPE angles of this token (the same for every head), once per tile
      float2 cs[16];
      if (kRope != kNoRope && t.kv && hf == 0) {
        const TokPos tp = token_pos(rope, valid ? n : 0);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int ax = pair_axis(j);
          const int pp = ax == 0 ? rope.t_offset + tp.t : (ax == 1 ? tp.h : tp.w);
          rope_cs_fast(pp, rope.inv_freq[j], cs[j].x, cs[j].y);
        }
      }
      bool ok = mbar_wait(&acc_full[buf], (tl >> 1) & 1, abort_flag, &g_qkv_error, kErrWait);
      if (!__all_sync(0xffffffffu, ok)) break;  // tcgen05.ld is warp-collective
      tc_fence_after();
      // key/value tile: the staging is free once every thread has finished
      // the previous tile's product
      if (t.kv) named_bar_sync(kBarEpi, kEpiThreads);
      __nv_bfloat16* qdst = Q + (static_cast<size_t>(t.b) * sc.N + (valid ? n : 0)) * sc.HD + f0;
      // the row's 128 features in four chunks of 32: bf16(acc + bias), then
      // straight to Q, or (keys) ReLU, key sums, RoPE, and to the staging
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        float v[32];
        tmem_ld_32x32b_x32(tmem + lane_base + buf * kAccCols + hf * 128 + ch * 32, v);
        uint32_t w[16];  // 32 features as bf16 pairs
        const bool in = f0 + ch * 32 < f_end;  // H*32 is a multiple of 32
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t bw[4] = {bq[ch & 1][k].x, bq[ch & 1][k].y, bq[ch & 1][k].z,
                                  bq[ch & 1][k].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            v[8 * k + 2 * e] += bf16_lo(bw[e]);
            v[8 * k + 2 * e + 1] += bf16_hi(bw[e]);
          }
        }
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = in && (valid || !t.kv) ? pack_bf16x2(v[2 * e], v[2 * e + 1]) : 0u;
        if (ch + 2 < 4) load_bias(ch + 2, bq[ch & 1]);
        if (!t.kv) {
          if (valid && in) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
              *reinterpret_cast<uint4*>(qdst + ch * 32 + 8 * k) =
                  make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
          }
          continue;
        }
        if (hf == 0) {
          // keys of head ch: ReLU (exact on bf16), the key sum of the
          // unrotated ReLU(k), then phi(k) = R(t, h, w) ReLU(k)
          float x[32];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            w[e] = relu_bf16x2(w[e]);
            x[2 * e] = bf16_lo(w[e]);
            x[2 * e + 1] = bf16_hi(w[e]);
          }
          zacc[ch] += warp_colsum(x, lane);
          if (kRope != kNoRope && valid) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float x0 = bf16_lo(w[j]), x1 = bf16_hi(w[j]);
              const float2 tt = __fmul2_rn(make_float2(x1, x1), make_float2(-cs[j].y, cs[j].x));
              const float2 yy = __ffma2_rn(make_float2(x0, x0), cs[j], tt);
              w[j] = pack_bf16x2(yy.x, yy.y);
            }
          }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k)
          st_shared_v4(stg + stg_offset(row, ch * 4 + k),
                       make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]));
      }
      // the accumulator may take the tile after next (CTA 0's barrier counts
      // one arrival per epilogue warp of the pair)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(acc_empty_0[buf]);
      if (!t.kv) continue;

      // ---- key/value tile: the staged rows are complete
      named_bar_sync(kBarEpi, kEpiThreads);
      // S[sh][16 smb + m][e] += sum over the tile's tokens of phi(k)[m] v[e]:
      // 8 steps of 16 tokens, A = phi(K)^T and B = V straight from the
      // staging rows (ldmatrix with transpose), fixed order
      {
        const int j = lane >> 3, q = lane & 7;
        const int a_dim = sh * 32 + smb * 16 + ((j & 1) << 3);  // A: matrix j = (m half, k half)
        const int a_row = ((j >> 1) << 3) + q;
        const int b_row = ((j & 1) << 3) + q;                    // B: matrix j = (k half, n block)
#pragma unroll
        for (int kb = 0; kb < kTokCta / 16; ++kb) {
          uint32_t a0, a1, a2, a3, b0, b1, b2, b3, b4, b5, b6, b7;
          ldsm_x4_trans(stg_k + stg_offset(kb * 16 + a_row, a_dim >> 3), a0, a1, a2, a3);
          ldsm_x4_trans(stg_v + stg_offset(kb * 16 + b_row, (sh * 32 + ((j >> 1) << 3)) >> 3), b0,
                        b1, b2, b3);
          ldsm_x4_trans(stg_v + stg_offset(kb * 16 + b_row, (sh * 32 + 16 + ((j >> 1) << 3)) >> 3),
                        b4, b5, b6, b7);
          mma_16816(sacc[0], a0, a1, a2, a3, b0, b1);
          mma_16816(sacc[1], a0, a1, a2, a3, b2, b3);
          mma_16816(sacc[2], a0, a1, a2, a3, b4, b5);
          mma_16816(sacc[3], a0, a1, a2, a3, b6, b7);
        }
      }

      if (t.last) {
        // ---- end of a run: this CTA's partial (S, z) of the run
        float* dst = part + ((static_cast<size_t>(t.b * sc.G + t.col) * sc.NK + t.k) * 2 + rank) *
                                kPartFloats;
        // accumulator nb: rows 16 smb + g (+ 8), columns 8 nb + 2 t4 (+ 1)
        float* ds = dst + sh * kD * kD + (smb * 16 + g) * kD + 2 * t4;
#pragma unroll
        for (int nb = 0; nb < 4; ++nb) {
          *reinterpret_cast<float2*>(ds + nb * 8) = make_float2(sacc[nb][0], sacc[nb][1]);
          *reinterpret_cast<float2*>(ds + 8 * kD + nb * 8) = make_float2(sacc[nb][2], sacc[nb][3]);
          sacc[nb][0] = sacc[nb][1] = sacc[nb][2] = sacc[nb][3] = 0.0f;
        }
        if (hf == 0) {
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            dst[kPartS + quad * 4 * kD + ch * kD + lane] = zacc[ch];
            zacc[ch] = 0.0f;
          }
        }
      }
    }
  }

  // neither CTA leaves while the other may still use its shared memory or
  // the pair's tensor memory
  tc_fence_before();
  __syncwarp();  // the cluster barrier is .aligned: whole warps
  cluster_sync_all();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kQkvTmemCols);
  }
}

// Sum of the partial slots of one (batch, head group) in a fixed order:
// chunk, slot, CTA of the pair, then (for z) TMEM lane quadrant. One thread
// per float4 of the result; a chunk's (at most 2 x 2) partials are loaded
// together, then added in that order.
constexpr int kCombineThreads = 128;
constexpr int kResultVec = (kPartS + 4 * kD) / 4;  // 1024 float4 of S, 32 of z

__global__ void __launch_bounds__(kCombineThreads)
qkv_combine(const QkvSched sc, const float* __restrict__ part, float* __restrict__ S,
            float* __restrict__ z) {
  pdl_wait();
  const int bg = blockIdx.x;
  const int b = bg / sc.G, g = bg - b * sc.G;
  const int v = blockIdx.y * kCombineThreads + threadIdx.x;
  if (v >= kResultVec) return;
  const bool is_s = v < kPartS / 4;
  constexpr int kVecPerPart = kPartFloats / 4;
  const float4* base =
      reinterpret_cast<const float4*>(part) + static_cast<size_t>(bg) * sc.NK * 2 * kVecPerPart;
  float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  // chunk by chunk, the two CTAs of the run's pair; a chunk's loads go together
  constexpr int kBatchK = 2;
  for (int k0 = 0; k0 < sc.NK; k0 += kBatchK) {
    float4 t[kBatchK][2][4];
#pragma unroll
    for (int kk = 0; kk < kBatchK; ++kk)
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int qd = 0; qd < 4; ++qd)
          if (k0 + kk < sc.NK && (!is_s || qd == 0))
            t[kk][j][qd] = __ldcg(base + (static_cast<size_t>(k0 + kk) * 2 + j) * kVecPerPart +
                                  (is_s ? v : kPartS / 4 + qd * kD + (v - kPartS / 4)));
#pragma unroll
    for (int kk = 0; kk < kBatchK; ++kk)
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int qd = 0; qd < 4; ++qd)
          if (k0 + kk < sc.NK && (!is_s || qd == 0)) {
            acc.x += t[kk][j][qd].x;
            acc.y += t[kk][j][qd].y;
            acc.z += t[kk][j][qd].z;
            acc.w += t[kk][j][qd].w;
          }
  }
  if (is_s) {
    const int hh = v / (kD * kD / 4), h = 4 * g + hh;
    if (h < sc.H)
      *reinterpret_cast<float4*>(S + (static_cast<size_t>(b) * sc.H + h) * kD * kD +
                                 (v - hh * (kD * kD / 4)) * 4) = acc;
  } else {
    const int w = v - kPartS / 4;  // head w / 8, dims 4 (w % 8) ..
    const int hh = w >> 3, h = 4 * g + hh;
    if (h < sc.H)
      *reinterpret_cast<float4*>(z + (static_cast<size_t>(b) * sc.H + h) * kD + (w & 7) * 4) = acc;
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
  s.NT = (N + kTokPair - 1) / kTokPair;
  s.G = (H + 3) / 4;
  s.QC = (s.HD + kCols - 1) / kCols;
  s.CT = s.G + s.QC;
  s.KB = (C + kKBlk - 1) / kKBlk;
  const long long total = 1LL * B * s.NT * s.CT;
  s.total = static_cast<int>(total);
  // Runs of L token tiles; the pairs take the runs in turn. L is the longest
  // run length whose load (the most tiles a pair gets) is within 3% of the
  // best over all L (short runs mean more partial states to write and sum).
  const int P = kNumSMs / 2;
  auto load = [&](int L) {
    const long long nk = (s.NT + L - 1) / L;
    const long long units = 1LL * B * nk * s.CT;
    return ((units + P - 1) / P) * L;  // tiles of the busiest pair (upper bound)
  };
  long long best = load(1);
  for (int L = 2; L <= s.NT; ++L) best = std::min(best, load(L));
  s.L = 1;
  for (int L = s.NT; L >= 1; --L)
    if (load(L) * 100 <= best * 103) {
      s.L = L;
      break;
    }
  s.NK = (s.NT + s.L - 1) / s.L;
  s.units = B * s.NK * s.CT;
  s.pairs = std::max(1, std::min(P, s.units));
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
  return static_cast<size_t>(B) * s.G * s.NK * 2 * kPartFloats;
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
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * sc.pairs, 1, 1);
  cfg.blockDim = dim3(kQkvThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(kQSmemBytes);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, kern, mx, mw, sc, p.rope,
                         static_cast<const __nv_bfloat16*>(bias), static_cast<__nv_bfloat16*>(Q),
                         part);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg2 = {};
  cfg2.gridDim = dim3(p.B * sc.G, (kResultVec + kCombineThreads - 1) / kCombineThreads, 1);
  cfg2.blockDim = dim3(kCombineThreads, 1, 1);
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
