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
// Warp roles (576 threads): warp 0 issues TMA loads, warp 1 allocates tensor
// memory and issues the MMAs (one elected lane), warps 2..17 transform tiles
// in shared memory and run the epilogue. Every mbarrier wait is bounded; a
// wait that gives up raises the library's device error word and the CTA
// drains its copies and MMAs and frees its tensor memory before returning.
#include <atomic>
#include <utility>

#include "la_tc_common.cuh"

namespace la {

// Device-wide error word: bit 0 = a bounded wait of a tensor-core kernel gave
// up. Read (and cleared) by la_device_error().
__device__ unsigned g_tc_error;

namespace {

using namespace sm100;

// ============================================================ the kernel

// One kernel template serves four launches: the state reduce alone, the
// apply alone, and the fused layer (reduce, a per-head-group hand-off, then
// apply) in two forms: the head group's CTAs as one thread-block cluster that
// hands the split partials over through distributed shared memory
// (kClusterLayer), or a cooperative grid that hands them over through global
// memory (kFusedLayer). A fifth launch, kChunkStates (bf16), is the reduce
// that writes the state of every 128-token chunk instead of one partial per
// split: the first step of token-causal attention (without RoPE it also writes
// the chunk's key sum; with RoPE the keys it holds are rotated and another
// kernel forms the key sums). All share
// one TMA stage ring of kNS stages (six; five
// in the cluster layer): a ring position p uses stage p % kNS with phase
// parity (p / kNS) & 1, whichever operation the tile belongs to.
enum Phases : int { kReduceOnly = 1, kApplyOnly = 2, kFusedLayer = 3, kClusterLayer = 7,
                    kChunkStates = 9 };

// Largest cluster of the cluster layer: the portable limit.
constexpr int kMaxCluster = 8;

constexpr int kMath = 512;                   // 16 math warps (warps 2..17)
constexpr int kThreadsTc = 64 + kMath;       // + TMA warp + MMA warp
constexpr int kApWG = kMath / 128;           // apply: at most 4 warpgroups, one tile each in turn
constexpr int kStageBytes = 32768;
constexpr int kRedT = 64;                    // reduce: tokens per stage (K and V, 4 heads)
constexpr int kRedBox = kRedT * 128;         // [64 tokens][64 dims] bf16
constexpr int kApT = 128;                    // apply: tokens per tile (Q, 4 heads)
constexpr int kApBox = kApT * 128;           // [128 tokens][64 dims] bf16
constexpr int kTmemCols = 512;               // reduce: cols [0,128); apply: one block per warpgroup

// The apply with and without RoPE. Without RoPE the denominators ReLU(q).z
// come from the tensor core too (an MMA against z, split into two bf16
// parts), so the transform of a Q tile is ReLU alone; the warpgroup's TMEM
// block then holds 4 x 32 numerator and 16 denominator columns, and three
// warpgroups fit the 512 columns. With RoPE the numerator needs the rotated
// phi(q) and the denominator the unrotated ReLU(q): the denominators are
// formed on the CUDA cores during the transform, and four warpgroups take
// tiles.
template <int kRope>
struct ApplyCfg {
  static constexpr bool kDenMma = kRope == kNoRope;
  static constexpr int kWG = kDenMma ? 3 : 4;            // warpgroups taking tiles
  static constexpr int kCols = kDenMma ? 160 : 128;      // TMEM columns per warpgroup
  static constexpr int kDenCol = 128;                    // first denominator column
};

// named barriers: 0 = whole CTA, 1 = all math threads, 2.. = apply warpgroups
constexpr int kBarMath = 1;
constexpr int kBarWG0 = 2;

// Shared-memory layout (byte offsets from the 1024-aligned base) for kNS
// stages of the ring; the RoPE table only with RoPE, the denominator operand
// only without, the partial-state buffer only in the cluster layer.
template <int kNS, bool kWithPart, bool kWithRope>
struct SmemLayout {
  static constexpr int stages = 0;
  // [16 warps][16] f32 key sums of the reduce; then the state S [4][32][32]
  // f32 that the apply uses
  static constexpr int zred = stages + kNS * kStageBytes;
  static constexpr int bop = zred + kGroupHeads * kD * kD * 4;  // [2 pairs][32 rows][128 B]
  // the apply's denominator operand: [2 boxes][16 rows][128 B] bf16, rows
  // 0-3 the heads' z (upper bf16 part), rows 4-7 the remainders
  static constexpr int zop = bop + 2 * 32 * 128;
  static constexpr int zs = zop + (kWithRope ? 0 : 2 * 16 * 128);  // [4][32] f32
  static constexpr int rope = zs + kGroupHeads * kD * 4;          // float2[kRopeTableMax]
  // cluster layer: this CTA's partial state, [4 heads][32*32 + 32] f32
  static constexpr int part = rope + (kWithRope ? kRopeTableMax * 8 : 0);
  static constexpr int bars = part + (kWithPart ? kGroupHeads * kStateFloats * 4 : 0);
  // full[kNS] empty[kNS] ready_a[kNS] ready_b[kNS] o_full[kNS] t_full[4]
  // t_empty[4] acc_full mma_done b_ready part_full done s_full
  static constexpr int nbars = 5 * kNS + 2 * kApWG + 6;
  static constexpr int misc = bars + nbars * 8;                // tmem base, abort, last flag
  static constexpr int bytes = misc + 16;
};

// Six stages of the ring in every launch but the cluster layer, whose
// partial-state buffer leaves room for five.
template <int kRope, int kPh>
struct LayerCfg {
  static constexpr int kNS = kPh == kClusterLayer ? 5 : 6;
  using Smem = SmemLayout<kNS, kPh == kClusterLayer, kRope != kNoRope>;
  static constexpr int kSmemBytes = Smem::bytes + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

struct LayerArgs {
  float* partials;     // [B*H][splits][kStateFloats]
  unsigned* arrive;    // [B*H] per head-group arrival counters (index b*H + h0)
  unsigned* ready;     // [B*H] fused layer: "combined state written" flags
  unsigned* depart;    // [B*H] fused layer: departure counters
  StateOut out;        // where the reduce's combined state goes
  const float* S_in;   // apply: state to apply (fused: out.out1_S)
  const float* z_in;
  int tiles_per_cta;   // apply: 128-token tiles per CTA
  int q_before_wait;   // apply only: Q may be read before the previous grid completes
  float* chunk_states; // kChunkStates: [B*H][nchunks][kStateFloats], chunk c's own (S, z)
  int nchunks;         // kChunkStates: ceil(N / 128)
};

template <int kRope, int kPh>
__global__ void __launch_bounds__(kThreadsTc, 1)
layer_tc(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
         const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_o,
         const Problem p, const RopeTable rt, const LayerArgs a) {
  constexpr bool kRed = (kPh & kReduceOnly) != 0;
  constexpr bool kApp = (kPh & kApplyOnly) != 0;
  constexpr bool kCl = kPh == kClusterLayer;
  constexpr bool kCh = kPh == kChunkStates;
  constexpr int kNS = LayerCfg<kRope, kPh>::kNS;
  using Smem = typename LayerCfg<kRope, kPh>::Smem;
  using AC = ApplyCfg<kRope>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Smem::bars);
  uint64_t* empty = full + kNS;
  uint64_t* ready_a = empty + kNS;  // reduce stage transformed: 512 arrivals
  uint64_t* ready_b = ready_a + kNS; // apply tile transformed: 128 arrivals
  uint64_t* o_full = ready_b + kNS;  // apply tile's O in the stage: 1 arrival
  uint64_t* t_full = o_full + kNS;   // [kApWG]
  uint64_t* t_empty = t_full + kApWG;   // [kApWG]
  uint64_t* acc_full = t_empty + kApWG;
  uint64_t* mma_done = acc_full + 1;
  uint64_t* b_ready = mma_done + 1;
  // cluster layer: every CTA's partial is in its shared memory / every CTA
  // is done reading this one's memory and the carry
  uint64_t* part_full = b_ready + 1;
  uint64_t* done = part_full + 1;
  uint64_t* s_full = done + 1;  // apply only: the state (S, z) copied in
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Smem::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Smem::misc + 4);
  volatile int* last_flag = reinterpret_cast<volatile int*>(smem + Smem::misc + 8);
  float* zred = reinterpret_cast<float*>(smem + Smem::zred);
  float* zs = reinterpret_cast<float*>(smem + Smem::zs);
  float2* rope_tab = reinterpret_cast<float2*>(smem + Smem::rope);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int group = blockIdx.y, b = blockIdx.z;
  const int h0 = group * kGroupHeads;
  const size_t cidx = static_cast<size_t>(b) * p.H + h0;
  // reduce work: the token split blockIdx.x, in 64-token stages
  const int n_begin = blockIdx.x * p.chunk;
  const int n_end = min(p.N, n_begin + p.chunk);
  const int nA = kRed && n_end > n_begin ? (n_end - n_begin + kRedT - 1) / kRedT : 0;
  // apply work: a range of 128-token tiles
  const int ntiles_all = (p.N + kApT - 1) / kApT;
  const int tile_begin = blockIdx.x * a.tiles_per_cta;
  const int nB = kApp ? max(0, min(ntiles_all, tile_begin + a.tiles_per_cta) - tile_begin) : 0;

  if (tid == 0) {
    for (int s = 0; s < kNS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&ready_a[s], kMath);
      mbar_init(&ready_b[s], 128);
      mbar_init(&o_full[s], 1);
    }
    for (int w = 0; w < kApWG; ++w) {
      mbar_init(&t_full[w], 1);
      // kChunkStates uses t_full/t_empty[0..1] for its two chunk accumulators;
      // t_empty then counts the four epilogue warps
      mbar_init(&t_empty[w], kCh ? 4 : 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(mma_done, 1);
    mbar_init(b_ready, 1);
    mbar_init(s_full, 1);
    if (kCl) {  // one arrival from each CTA of the cluster
      mbar_init(part_full, gridDim.x);
      mbar_init(done, gridDim.x);
    }
    *abort_flag = 0;
    *last_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == 0 && lane == 0) {
    if (kRed) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
    }
    if (kApp) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_o);
    }
  }
  if (kRope == kRopeTable && tid >= 64) build_rope_table(p.rope, rope_tab, tid - 64, kMath);
  if (kCh && kRope == kNoRope && tid >= 64 && tid < 64 + 256) {
    // a 4 KB tile of bf16 ones: the B operand whose product with phi(K)^T is
    // the key sum of every dim (with RoPE the keys in shared memory are
    // rotated, so the chunks' key sums are formed by another kernel)
    st_shared_v4(smem_u32(smem + Smem::zop) + (tid - 64) * 16,
                 make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u));
    fence_proxy_async_smem();
  }
  __syncthreads();
  // cluster layer: every CTA's barriers are initialised before any other CTA
  // may arrive on them
  if (kCl) cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(smem);

  // Programmatic dependent launch: global memory is touched only after the
  // previous grid has completed -- except Q in an apply whose previous grid is
  // this library's own reduce (q_before_wait), which the TMA warp may fetch
  // early. The next grid may then be scheduled.
  const bool early_q = kPh == kApplyOnly && a.q_before_wait;
  if (!(warp == 0 && early_q)) pdl_wait();
  if (tid == 64) pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA loads
    if (lane == 0) {
      int pos = 0;
      bool ok = true;
      for (int i = 0; ok && i < nA; ++i, ++pos) {
        const int s = pos % kNS;
        if (!(ok = mbar_wait(&empty[s], ((pos / kNS) & 1) ^ 1, abort_flag, &g_tc_error,
                             kErrWait)))
          break;
        mbar_arrive_expect_tx(&full[s], kStageBytes);
        uint8_t* st = smem + Smem::stages + s * kStageBytes;
        const int y = n_begin + i * kRedT;
        tma_load_3d(st, &tm_k, &full[s], h0 * 32, y, b);
        tma_load_3d(st + kRedBox, &tm_k, &full[s], h0 * 32 + 64, y, b);
        tma_load_3d(st + 2 * kRedBox, &tm_v, &full[s], h0 * 32, y, b);
        tma_load_3d(st + 3 * kRedBox, &tm_v, &full[s], h0 * 32 + 64, y, b);
      }
      // Q tiles. A stage last used by an apply tile is handed back by this
      // thread: once that tile's O is in the stage (o_full), it stores it
      // with TMA, waits until the store has read the stage, releases the
      // stage (empty: the warpgroups' phase guard waits on it) and reloads
      // it. The warpgroups never wait for their stores.
      auto store_tile = [&](int q) -> bool {  // q: apply tile index
        const int qs = (nA + q) % kNS;
        if (!mbar_wait(&o_full[qs], (q / kNS) & 1, abort_flag, &g_tc_error, kErrWait))
          return false;
        uint8_t* tile = smem + Smem::stages + qs * kStageBytes;
        const int n0 = (tile_begin + q) * kApT;
        tma_store_3d(&tm_o, tile, h0 * 32, n0, b);
        tma_store_3d(&tm_o, tile + kApBox, h0 * 32 + 64, n0, b);
        bulk_commit();
        bulk_wait_read<0>();
        mbar_arrive(&empty[qs]);
        return true;
      };
      // apply only: the state (S, z) of the group's heads, one bulk copy
      // each, issued ahead of the Q tiles so that it does not queue behind
      // them; when Q may be read before the previous grid completes, after
      // the first ring of Q tiles and the wait for that grid
      const int sheads = kApp ? max(0, min(kGroupHeads, p.H - h0)) : 0;
      bool state_issued = kPh != kApplyOnly;
      auto issue_state = [&]() {
        mbar_arrive_expect_tx(s_full, sheads * (kD * kD + kD) * 4);
        if (sheads > 0) {
          bulk_load(smem + Smem::zred, a.S_in + cidx * kD * kD, sheads * kD * kD * 4, s_full);
          bulk_load(smem + Smem::zs, a.z_in + cidx * kD, sheads * kD * 4, s_full);
        }
        state_issued = true;
      };
      if (!state_issued && !early_q) issue_state();
      int stored = 0;  // apply tiles whose O has been stored
      for (int i = 0; ok && i < nB; ++i, ++pos) {
        const int s = pos % kNS;
        if (i >= kNS) {  // the stage's previous tile was apply tile i - kNS
          if (!(ok = store_tile(i - kNS))) break;
          ++stored;
        } else if (!(ok = mbar_wait(&empty[s], ((pos / kNS) & 1) ^ 1, abort_flag, &g_tc_error,
                                    kErrWait))) {
          break;
        }
        mbar_arrive_expect_tx(&full[s], kStageBytes);
        uint8_t* st = smem + Smem::stages + s * kStageBytes;
        const int y = (tile_begin + i) * kApT;
        tma_load_3d(st, &tm_q, &full[s], h0 * 32, y, b);
        tma_load_3d(st + kApBox, &tm_q, &full[s], h0 * 32 + 64, y, b);
        if (!state_issued && i + 1 == min(kNS, nB)) {
          pdl_wait();
          issue_state();
        }
      }
      if (!state_issued) {  // (only when the loop stopped early)
        pdl_wait();
        issue_state();
      }
      for (int q = stored; ok && q < nB; ++q) ok = store_tile(q);
      // drain: every load issued must have landed, and every store completed,
      // before the CTA exits
      for (int q = max(0, pos - kNS); q < pos; ++q)
        mbar_drain(&full[q % kNS], (q / kNS) & 1, &g_tc_error, kErrWait);
      bulk_wait<0>();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      int pos = 0;
      bool ok = true;
      const uint32_t id_red = idesc_bf16_f32(128, 128, 1, 1);
      const uint32_t id_z = idesc_bf16_f32(128, 16, 1, 1);
      const uint64_t ones_d = smem_desc_sw128(sbase + Smem::zop, 2048, 1024);
      for (int i = 0; i < nA; ++i, ++pos) {
        const int s = pos % kNS;
        // kChunkStates: chunk c = stages 2c, 2c + 1 accumulates in TMEM block
        // c & 1 (state in 128 columns, key sums in the next 16), afresh
        const int c = i >> 1, cb = c & 1;
        const bool first = (i & 1) == 0;
        if (kCh && first &&
            !(ok = mbar_wait(&t_empty[cb], ((c >> 1) & 1) ^ 1, abort_flag, &g_tc_error, kErrWait)))
          break;
        if (!(ok = mbar_wait(&ready_a[s], (i / kNS) & 1, abort_flag, &g_tc_error, kErrWait)))
          break;
        tc_fence_after();
        const uint32_t st = sbase + Smem::stages + s * kStageBytes;
        const uint32_t acc = kCh ? tmem + cb * 160 : tmem;
        // 16 tokens = two 8-row groups of 128 bytes; LBO = the second 64-dim box
        const uint64_t a0 = smem_desc_sw128(st, kRedBox, 1024);
        const uint64_t b0 = smem_desc_sw128(st + 2 * kRedBox, kRedBox, 1024);
#pragma unroll
        for (int kk = 0; kk < kRedT / 16; ++kk) {
          const uint64_t ad = desc_at(a0, kk * 2048);
          const uint64_t bd = desc_at(b0, kk * 2048);
          const uint32_t accum = kCh ? ((first && kk == 0) ? 0u : 1u) : ((i > 0 || kk > 0) ? 1u : 0u);
          mma_bf16(acc, ad, bd, id_red, accum);
          if (kCh && kRope == kNoRope) mma_bf16(acc + 128, ad, ones_d, id_z, accum);  // key sums
        }
        mma_commit(&empty[s]);
        if (kCh && (!first || i == nA - 1)) mma_commit(&t_full[cb]);
      }
      if (kRed) mma_commit(acc_full);
      if (ok && kApp && nB > 0) ok = mbar_wait(b_ready, 0, abort_flag, &g_tc_error, kErrWait);
      const uint32_t id_ap = idesc_bf16_f32(128, 32, 0, 0);
      const uint32_t id_den = idesc_bf16_f32(128, 16, 0, 0);
      const uint64_t bop0 = smem_desc_sw128(sbase + Smem::bop, 16, 1024);
      const uint64_t zop0 = smem_desc_sw128(sbase + Smem::zop, 16, 1024);
      for (int j = 0; ok && j < nB; ++j, ++pos) {
        const int s = pos % kNS;
        const int w = j % AC::kWG;
        if (!(ok = mbar_wait(&ready_b[s], (j / kNS) & 1, abort_flag, &g_tc_error, kErrWait)))
          break;
        if (!(ok = mbar_wait(&t_empty[w], ((j / AC::kWG) & 1) ^ 1, abort_flag, &g_tc_error,
                             kErrWait)))
          break;
        tc_fence_after();
        const uint32_t acc = tmem + w * AC::kCols;
        const uint64_t q0 = smem_desc_sw128(sbase + Smem::stages + s * kStageBytes, 16, 1024);
#pragma unroll
        for (int hh = 0; hh < kGroupHeads; ++hh) {
          const uint32_t koff = (hh & 1) * 64;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            const uint64_t ad = desc_at(q0, (hh >> 1) * kApBox + koff + kk * 32);
            const uint64_t bd = desc_at(bop0, (hh >> 1) * 4096 + koff + kk * 32);
            mma_bf16(acc + hh * 32, ad, bd, id_ap, kk);
          }
        }
        if (AC::kDenMma) {
          // the denominators: ReLU(Q) (all 128 dims) times the z operand
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t ad = desc_at(q0, (kk >> 2) * kApBox + (kk & 3) * 32);
            const uint64_t bd = desc_at(zop0, (kk >> 2) * 2048 + (kk & 3) * 32);
            mma_bf16(acc + AC::kDenCol, ad, bd, id_den, kk > 0 ? 1u : 0u);
          }
        }
        mma_commit(&t_full[w]);
      }
      mma_commit(mma_done);
      mbar_drain(mma_done, 0, &g_tc_error, kErrWait);
    }
  } else {
    // ---------------------------------------------------------- math warps
    const int mt = tid - 64;
    bool alive = true;
    if (kRed) {
      // feature map of K, key sum. Math warp wi owns, in every 64-token
      // stage, the rows 32 (wi >> 3) + lane of head (wi >> 1) & 3 of the
      // group, dims [16 half, 16 half + 16) with half = wi & 1: two 16-byte
      // chunks of one row per thread, so a warp reads 32 rows of one chunk
      // column (conflict-free under the 128-byte swizzle) and which RoPE
      // pairs a thread rotates is fixed per warp.
      const int wi = mt >> 5;
      const int half = wi & 1, hq = (wi >> 1) & 3;
      const int rg = (wi >> 3) * 32 + lane;
      const int cc0 = (hq & 1) * 4 + half * 2;  // first of the two chunks in the 128-byte row
      float2 zacc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) zacc[e] = make_float2(0.0f, 0.0f);
      TokPos tp = {0, 0, 0};
      if (kRope != kNoRope) tp = token_pos(p.rope, n_begin + rg);
      // kChunkStates: warps 2..5 (TMEM lane quadrant q = head q of the group)
      // copy each finished chunk's (S, z) from TMEM to the chunk-state buffer,
      // one stage after the chunk's last stage so its MMAs are done by then
      const int nch = (nA + 1) / 2;
      int next_chunk = 0;
      auto chunk_epilogue = [&](int c) {
        const int q = warp & 3, cb = c & 1;
        bool got = mbar_wait(&t_full[cb], (c >> 1) & 1, abort_flag, &g_tc_error, kErrWait);
        got = __all_sync(0xffffffffu, got);  // tcgen05.ld is warp-collective
        float v[32], zv[8];
        if (got) {
          tc_fence_after();
          const uint32_t base = tmem + (static_cast<uint32_t>(32 * q) << 16) + cb * 160;
          tmem_ld_32x32b_x32(base + 32 * q, v);
          if (kRope == kNoRope) tmem_ld_32x32b_x8(base + 128, zv);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&t_empty[cb]);
        if (got && h0 + q < p.H) {
          float* dst = a.chunk_states +
                       ((cidx + q) * a.nchunks + n_begin / kTileTokens + c) * kStateFloats;
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + lane * kD + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
          if (kRope == kNoRope) dst[kD * kD + lane] = zv[0];
        }
      };
      for (int i = 0; i < nA; ++i) {
        const int s = i % kNS;
        if (!mbar_wait(&full[s], (i / kNS) & 1, abort_flag, &g_tc_error, kErrWait)) {
          alive = false;
          break;
        }
        const uint32_t kb = sbase + Smem::stages + s * kStageBytes + (hq >> 1) * kRedBox;
        const uint32_t a0 = kb + sw128_offset(rg, cc0), a1 = kb + sw128_offset(rg, cc0 + 1);
        uint4 u0 = ld_shared_v4(a0), u1 = ld_shared_v4(a1);
        u0.x = relu_bf16x2(u0.x);
        u0.y = relu_bf16x2(u0.y);
        u0.z = relu_bf16x2(u0.z);
        u0.w = relu_bf16x2(u0.w);
        u1.x = relu_bf16x2(u1.x);
        u1.y = relu_bf16x2(u1.y);
        u1.z = relu_bf16x2(u1.z);
        u1.w = relu_bf16x2(u1.w);
        float x[16];
        {
          float xa[8], xb[8];
          unpack8(u0, xa);
          unpack8(u1, xb);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            x[e] = xa[e];
            x[8 + e] = xb[e];
          }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e)
          zacc[e] = __fadd2_rn(zacc[e], make_float2(x[2 * e], x[2 * e + 1]));
        if (kRope != kNoRope) {
          if (n_begin + i * kRedT + rg < p.N) {
            float2 cs[8];
            if (kRope == kRopeTable) {
              const RopeBases rb = rope_bases(p.rope, tp);
              if (half == 0) rope_table8<0>(rope_tab, rb, cs);
              else rope_table8<1>(rope_tab, rb, cs);
            } else {
              if (half == 0) rope_fly8<0>(p.rope, tp, cs);
              else rope_fly8<1>(p.rope, tp, cs);
            }
            rotate8(x, cs);
            float xa[8], xb[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              xa[e] = x[e];
              xb[e] = x[8 + e];
            }
            u0 = pack8(xa);
            u1 = pack8(xb);
          }
          token_pos_advance(p.rope, tp, kRedT);
        }
        st_shared_v4(a0, u0);
        st_shared_v4(a1, u1);
        fence_proxy_async_smem();
        mbar_arrive(&ready_a[s]);
        if (kCh && warp >= 2 && warp < 6) {
          // chunk c ends at stage min(2c + 1, nA - 1)
          while (next_chunk < nch && min(2 * next_chunk + 1, nA - 1) <= i - 1)
            chunk_epilogue(next_chunk++);
        }
      }
      if (kCh) {
        if (warp >= 2 && warp < 6 && alive)
          while (next_chunk < nch) chunk_epilogue(next_chunk++);
        alive = !bar_any(kBarMath, kMath, !alive || *abort_flag);
      }
      if (!kCh) {
      {
        // the warp's 16 key sums over its 32 rows (fixed butterfly order);
        // lane 0 leaves them in zred[wi][16]
        float zv[16];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          zv[2 * e] = zacc[e].x;
          zv[2 * e + 1] = zacc[e].y;
        }
#pragma unroll
        for (int w = 16; w >= 1; w >>= 1)
#pragma unroll
          for (int e = 0; e < 16; ++e) zv[e] += __shfl_xor_sync(0xffffffffu, zv[e], w);
        if (lane == 0) {
#pragma unroll
          for (int e = 0; e < 16; e += 4)
            *reinterpret_cast<float4*>(zred + wi * 16 + e) = make_float4(zv[e], zv[e + 1], zv[e + 2], zv[e + 3]);
        }
      }
      alive = !bar_any(kBarMath, kMath, !alive || *abort_flag);
      // state of the four heads: the 32x32 diagonal blocks of the accumulator
      if (warp >= 2 && warp < 6) {
        const int q = warp & 3;  // TMEM lane quadrant = head in the group
        float v[32];
        bool got = alive && nA > 0 && mbar_wait(acc_full, 0, abort_flag, &g_tc_error, kErrWait);
        got = __all_sync(0xffffffffu, got);  // tcgen05.ld is warp-collective
        if (got) {
          tc_fence_after();
          tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(32 * q) << 16) + 32 * q, v);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0.0f;
        }
        const int h = h0 + q;
        if (kCl || h < p.H) {
          float* dst = kCl ? reinterpret_cast<float*>(smem + Smem::part) + q * kStateFloats + lane * kD
                           : a.partials + ((cidx + q) * p.splits + blockIdx.x) * kStateFloats + lane * kD;
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        }
      }
      if (mt < 128) {
        // key sum of dim mt of the group: the two row groups' warp sums, in order
        const int q = mt >> 5, d = mt & 31;
        const int wq = q * 2 + (d >> 4);  // warp (of row group 0) holding this dim
        const float sum = zred[wq * 16 + (d & 15)] + zred[(8 + wq) * 16 + (d & 15)];
        if (kCl)
          reinterpret_cast<float*>(smem + Smem::part)[q * kStateFloats + kD * kD + d] = sum;
        else if (h0 + q < p.H)
          a.partials[((cidx + q) * p.splits + blockIdx.x) * kStateFloats + kD * kD + d] = sum;
      }
      }  // !kCh
      tc_fence_before();
    }

    float* sbuf = zred;  // [4][32][32] f32: the state for the apply, free once the reduce is done
    if (kCl) {
      // ---- hand-off inside the cluster (the head group's token splits, one
      // CTA each; cluster rank = split index). Once every CTA's partial is in
      // its shared memory, every CTA sums all of them in split order, plus the
      // carry, straight into its own shared memory (the loads of all splits
      // are issued before the sum): the sums are those of the reduce-only
      // launch's combine, bit for bit. The state is written out at the end,
      // once no CTA reads the carry any more (it may be updated in place).
      named_bar_sync(kBarMath, kMath);  // this CTA's partial is in Smem::part
      const uint32_t ncta = gridDim.x;
      if (mt == 0) {
        fence_acq_rel_cluster();
        for (uint32_t r = 0; r < ncta; ++r) mbar_arrive_remote(mapa_shared(smem_u32(part_full), r));
      }
      bool ok = alive && mbar_wait_cluster(part_full, 0, abort_flag, &g_tc_error, kErrWait);
      constexpr int kVec = kStateFloats / 4;  // float4 per head
      const int heads = min(kGroupHeads, p.H - h0);
      const uint32_t part_s = sbase + Smem::part;
      if (ok) {
        for (int v = mt; v < kGroupHeads * kVec; v += kMath) {
          float4 t[kMaxCluster];
#pragma unroll
          for (int r = 0; r < kMaxCluster; ++r)
            if (r < static_cast<int>(ncta)) t[r] = ld_cluster_v4(mapa_shared(part_s + v * 16, r));
          float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
          for (int r = 0; r < kMaxCluster; ++r)
            if (r < static_cast<int>(ncta)) {
              acc.x += t[r].x;
              acc.y += t[r].y;
              acc.z += t[r].z;
              acc.w += t[r].w;
            }
          const int hh = v / kVec, i = (v - hh * kVec) * 4;
          const bool is_s = i < kD * kD;
          if (hh < heads) {
            const size_t bh = cidx + hh;
            const float* c = is_s ? a.out.carry_S : a.out.carry_z;
            if (c != nullptr) {
              const float4 cv = *reinterpret_cast<const float4*>(
                  c + (is_s ? bh * kD * kD + i : bh * kD + (i - kD * kD)));
              acc = make_float4(cv.x + acc.x, cv.y + acc.y, cv.z + acc.z, cv.w + acc.w);
            }
          }
          *reinterpret_cast<float4*>(is_s ? sbuf + hh * kD * kD + i : zs + hh * kD + (i - kD * kD)) =
              acc;
        }
      }
      alive = !bar_any(kBarMath, kMath, !ok || *abort_flag);
      // no more reads of other CTAs' shared memory, nor of the carry
      if (mt == 0)
        for (uint32_t r = 0; r < ncta; ++r) mbar_arrive_remote(mapa_shared(smem_u32(done), r));
    }
    if (kRed && !kCl && !kCh) {
      // ---- second phase of the reduce. The named barrier orders each math
      // thread's partial stores before the release fence of the arriving
      // thread.
      named_bar_sync(kBarMath, kMath);
      if (mt == 0) {
        fence_acq_rel_gpu();
        const unsigned prev = atomicAdd(&a.arrive[cidx], 1u);
        *last_flag = prev == gridDim.x - 1;
        if (kPh == kFusedLayer) {
          // single-launch layer: every CTA of the head group waits for all the
          // splits' partials (the launch is cooperative: all CTAs are resident)
          spin_count(&a.arrive[cidx], gridDim.x, abort_flag, &g_tc_error);
        } else if (*last_flag) {
          fence_acq_rel_gpu();
        }
      }
      named_bar_sync(kBarMath, kMath);
      const bool last = *last_flag != 0;
      if (kPh == kReduceOnly) {
        // the CTA that arrived last sums every split's partial in split order
        // (+ carry) and writes the state
        const bool wanted = a.out.out1_S != nullptr || a.out.out1_z != nullptr ||
                            a.out.out2_S != nullptr || a.out.out2_z != nullptr;
        const int heads = min(kGroupHeads, p.H - h0);
        const uint32_t pbytes =
            static_cast<uint32_t>(heads) * static_cast<uint32_t>(p.splits) * kStateFloats * 4u;
        if (last && alive && wanted && pbytes <= static_cast<uint32_t>(kNS) * kStageBytes) {
          // The group's partials are contiguous in the workspace: one bulk
          // copy brings them all into the idle stage ring (every load has
          // landed and every MMA has read its stage), then each thread sums
          // its columns over the splits from shared memory.
          if (mt == 0) {
            fence_proxy_async_global();  // after the acquire above
            mbar_arrive_expect_tx(s_full, pbytes);
            bulk_load(smem + Smem::stages, a.partials + cidx * p.splits * kStateFloats, pbytes,
                      s_full);
          }
          if (mbar_wait(s_full, 0, abort_flag, &g_tc_error, kErrWait)) {
            const float* ps = reinterpret_cast<const float*>(smem + Smem::stages);
            constexpr int kVec = kStateFloats / 4;
            for (int v = mt; v < heads * kVec; v += kMath) {
              const int hh = v / kVec, i = (v - hh * kVec) * 4;
              float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
              for (int s2 = 0; s2 < p.splits; ++s2) {
                const float4 t = *reinterpret_cast<const float4*>(
                    ps + (static_cast<size_t>(hh) * p.splits + s2) * kStateFloats + i);
                acc.x += t.x;
                acc.y += t.y;
                acc.z += t.z;
                acc.w += t.w;
              }
              const bool is_s = i < kD * kD;
              const size_t bh = cidx + hh;
              const size_t o = is_s ? bh * kD * kD + i : bh * kD + (i - kD * kD);
              const float* c = is_s ? a.out.carry_S : a.out.carry_z;
              if (c != nullptr) {
                const float4 cv = *reinterpret_cast<const float4*>(c + o);
                acc = make_float4(cv.x + acc.x, cv.y + acc.y, cv.z + acc.z, cv.w + acc.w);
              }
              float* d1 = is_s ? a.out.out1_S : a.out.out1_z;
              float* d2 = is_s ? a.out.out2_S : a.out.out2_z;
              if (d1 != nullptr) *reinterpret_cast<float4*>(d1 + o) = acc;
              if (d2 != nullptr) *reinterpret_cast<float4*>(d2 + o) = acc;
            }
          }
        } else if (last && alive && wanted) {
          combine_from_global<kMath>(p, b, h0, mt, a.partials, a.out);
        }
        named_bar_sync(kBarMath, kMath);
        if (mt == 0 && last) a.arrive[cidx] = 0u;  // ready for the next call
      } else {
        // single-launch layer: every CTA sums the partials itself, in the same
        // order as the reduce-only launch, straight into shared memory (so the
        // results are bitwise those of reduce + apply); the state is written
        // out by the last CTA to leave, once every CTA has read the carry
        if (*abort_flag) alive = false;
        const int heads = min(kGroupHeads, p.H - h0);
        for (int i = mt; i < (kGroupHeads - heads) * (kD * kD + kD); i += kMath) {
          const int hh = heads + i / (kD * kD + kD), k = i % (kD * kD + kD);
          if (k < kD * kD) sbuf[hh * kD * kD + k] = 0.0f;
          else zs[hh * kD + k - kD * kD] = 0.0f;
        }
        const StateOut carry_only = {a.out.carry_S, a.out.carry_z, nullptr, nullptr, nullptr,
                                     nullptr};
        if (alive) combine_from_global<kMath>(p, b, h0, mt, a.partials, carry_only, sbuf, zs);
        named_bar_sync(kBarMath, kMath);
      }
    }

    if (kApp && alive) {
      // ---- the state of the four heads as the MMA's B operand: row e of head
      // pair j holds S[h][0..31][e] of heads 2j and 2j+1 in bf16 (K-major,
      // 128-byte swizzle); S goes through shared memory with 16-byte loads
      if (kPh == kApplyOnly) {  // the fused layer has it in shared memory already
        // the TMA warp copies the group's heads in; heads beyond H are zero
        const int heads = min(kGroupHeads, p.H - h0);
        for (int idx = heads * kD * kD / 4 + mt; idx < kGroupHeads * kD * kD / 4; idx += kMath)
          *reinterpret_cast<float4*>(sbuf + idx * 4) = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (mt >= heads * kD && mt < kGroupHeads * kD) zs[mt] = 0.0f;
        const bool got = mbar_wait(s_full, 0, abort_flag, &g_tc_error, kErrWait);
        if (bar_any(kBarMath, kMath, !got || *abort_flag)) alive = false;
      }
      {
        const int idx = mt;  // 2 pairs x 32 rows x 8 chunks = 512 = kMath
        const int j = idx >> 8, e = (idx >> 3) & 31, c = idx & 7;
        const int hh = 2 * j + (c >> 2), d0 = (c & 3) * 8;
        float x[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) x[k] = sbuf[hh * kD * kD + (d0 + k) * kD + e];
        st_shared_v4(sbase + Smem::bop + j * 4096 + sw128_offset(e, c), pack8(x));
      }
      if (AC::kDenMma && mt < 256) {
        // the denominator operand (K-major, 2 boxes x 16 rows x 128 B): row
        // hh < 4 holds bf16(z) of head hh in the head's 32 dims, row 4 + hh
        // the remainder z - bf16(z), rounded to bf16; everything else is 0,
        // so column hh + 4 t of the MMA's result is ReLU(q) . (part t of z)
        const int box = mt >> 7, r = (mt >> 3) & 15, c = mt & 7;
        const int hh = 2 * box + (c >> 2), d0 = (c & 3) * 8;
        float x[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float zv = zs[hh * kD + d0 + k];
          const float hi = __bfloat162float(__float2bfloat16_rn(zv));
          x[k] = (r & 3) != hh || r >= 8 ? 0.0f : (r < 4 ? hi : zv - hi);
        }
        st_shared_v4(sbase + Smem::zop + box * 2048 + sw128_offset(r, c), pack8(x));
      }
      fence_proxy_async_smem();
      named_bar_sync(kBarMath, kMath);
      if (mt == 0) mbar_arrive(b_ready);
      // ---- apply: warpgroup wg < AC::kWG owns tiles wg, wg + kWG, ...;
      // thread = token row
      const int wg = (warp - 2) >> 2;
      const int quad = warp & 3;
      const int row = quad * 32 + lane;
      const bool leader = (warp == 2 + 4 * wg) && lane == 0;
      for (int j = wg; wg < AC::kWG && j < nB; j += AC::kWG) {
        const int pos = nA + j;
        const int s = pos % kNS;
        // The stage's previous apply tile (pos - kNS) belonged to another
        // warpgroup. A parity wait cannot tell phase k from k + 2, so wait for
        // that tile's release first: then the full phase awaited next is
        // unambiguous. (Every earlier release precedes the load of this
        // warpgroup's previous tile, which it has already consumed.)
        bool ok = true;
        if (pos - kNS >= nA)
          ok = mbar_wait(&empty[s], ((pos - kNS) / kNS) & 1, abort_flag, &g_tc_error,
                         kErrWait);
        ok = ok && mbar_wait(&full[s], (pos / kNS) & 1, abort_flag, &g_tc_error, kErrWait);
        if (bar_any(kBarWG0 + wg, 128, !ok || *abort_flag)) break;
        const int n0 = (tile_begin + j) * kApT;
        const int n = n0 + row;
        float2 cs[16];
        if (kRope != kNoRope) {
          const TokPos tp = token_pos(p.rope, min(n, p.N - 1));
          float2 c0[8], c1[8];
          if (kRope == kRopeTable) {
            const RopeBases rb = rope_bases(p.rope, tp);
            rope_table8<0>(rope_tab, rb, c0);
            rope_table8<1>(rope_tab, rb, c1);
          } else {
            rope_fly8<0>(p.rope, tp, c0);
            rope_fly8<1>(p.rope, tp, c1);
          }
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            cs[jj] = c0[jj];
            cs[8 + jj] = c1[jj];
          }
        }
        float den[kGroupHeads] = {0.0f, 0.0f, 0.0f, 0.0f};
        const uint32_t st = sbase + Smem::stages + s * kStageBytes;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int hh = c >> 2, d0 = (c & 3) * 8;
          const uint32_t addr = st + (c >> 3) * kApBox + sw128_offset(row, c & 7);
          uint4 u = ld_shared_v4(addr);
          u.x = relu_bf16x2(u.x);
          u.y = relu_bf16x2(u.y);
          u.z = relu_bf16x2(u.z);
          u.w = relu_bf16x2(u.w);
          if (AC::kDenMma) {  // ReLU is the whole transform
            st_shared_v4(addr, u);
            continue;
          }
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
        mbar_arrive(&ready_b[s]);

        // epilogue: O = num / den over the tile in shared memory (the MMA has
        // read it); the TMA warp stores it and hands the stage back
        ok = mbar_wait(&t_full[wg], (j / AC::kWG) & 1, abort_flag, &g_tc_error, kErrWait);
        tc_fence_after();
        if (bar_any(kBarWG0 + wg, 128, !ok || *abort_flag)) break;
        const uint32_t acc = tmem + (static_cast<uint32_t>(quad * 32) << 16) + wg * AC::kCols;
        if (AC::kDenMma) {
          float dv[8];
          tmem_ld_32x32b_x8(acc + AC::kDenCol, dv);
#pragma unroll
          for (int hh = 0; hh < kGroupHeads; ++hh) den[hh] = dv[hh] + dv[4 + hh];
        }
#pragma unroll
        for (int hh = 0; hh < kGroupHeads; ++hh) {
          float v[32];
          tmem_ld_32x32b_x32(acc + hh * 32, v);
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
        fence_proxy_async_smem();
        named_bar_sync(kBarWG0 + wg, 128);
        if (leader) {
          mbar_arrive(&t_empty[wg]);
          mbar_arrive(&o_full[s]);  // the TMA warp stores the tile
        }
      }
    }
    if (kCl) {
      // The CTA's shared memory must outlive the other CTAs' reads of it, and
      // the carry may be overwritten only once every CTA has read it: wait
      // until every CTA of the cluster is done (not stopped by an abort: the
      // other CTAs read this one's memory regardless), then write slice
      // `rank` of the combined state out.
      if (mt == 0 && !mbar_try_wait_acq_cluster(done, 0)) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait_acq_cluster(done, 0)) {
          if (globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicOr(&g_tc_error, kErrWait);
            *abort_flag = 1;
            break;
          }
        }
      }
      named_bar_sync(kBarMath, kMath);
      if (alive && !*abort_flag) {
        constexpr int kVec = kStateFloats / 4;
        const int heads = min(kGroupHeads, p.H - h0);
        const int nv = heads * kVec;
        const int per = (nv + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x);
        const int v_lo = static_cast<int>(cluster_ctarank()) * per;
        for (int v = v_lo + mt; v < min(nv, v_lo + per); v += kMath) {
          const int hh = v / kVec, i = (v - hh * kVec) * 4;
          const bool is_s = i < kD * kD;
          const size_t bh = cidx + hh;
          const size_t o = is_s ? bh * kD * kD + i : bh * kD + (i - kD * kD);
          const float4 val = *reinterpret_cast<const float4*>(
              is_s ? sbuf + hh * kD * kD + i : zs + hh * kD + (i - kD * kD));
          float* d1 = is_s ? a.out.out1_S : a.out.out1_z;
          float* d2 = is_s ? a.out.out2_S : a.out.out2_z;
          if (d1 != nullptr) *reinterpret_cast<float4*>(d1 + o) = val;
          if (d2 != nullptr) *reinterpret_cast<float4*>(d2 + o) = val;
        }
      }
    }
    if (kPh == kFusedLayer) {
      // every CTA has read the carry and the partials once all have reached
      // this point: the last to arrive here writes the state out (the carry
      // may be updated in place) and resets the group's words
      if (mt == 0) {
        fence_acq_rel_gpu();
        const unsigned prev = atomicAdd(&a.depart[cidx], 1u);
        *last_flag = prev == gridDim.x - 1;
        if (*last_flag) fence_acq_rel_gpu();
      }
      named_bar_sync(kBarMath, kMath);
      if (*last_flag) {
        const int heads = min(kGroupHeads, p.H - h0);
        for (int i = mt; i < heads * (kD * kD + kD) / 4; i += kMath) {
          const int hh = i / ((kD * kD + kD) / 4), k = (i % ((kD * kD + kD) / 4)) * 4;
          const bool is_s = k < kD * kD;
          const float4 v = is_s ? *reinterpret_cast<const float4*>(sbuf + hh * kD * kD + k)
                                : *reinterpret_cast<const float4*>(zs + hh * kD + k - kD * kD);
          const size_t o = is_s ? (cidx + hh) * kD * kD + k : (cidx + hh) * kD + k - kD * kD;
          float* d1 = is_s ? a.out.out1_S : a.out.out1_z;
          float* d2 = is_s ? a.out.out2_S : a.out.out2_z;
          if (d1 != nullptr) *reinterpret_cast<float4*>(d1 + o) = v;
          if (d2 != nullptr) *reinterpret_cast<float4*>(d2 + o) = v;
        }
        if (mt == 0) {
          a.arrive[cidx] = 0u;
          a.depart[cidx] = 0u;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Health check of the bounded waits: one warp waits for a barrier phase that
// nothing completes; the wait gives up after limit_ns and raises the error
// word, exactly as a stalled pipeline stage of the kernels above would.
__global__ void __launch_bounds__(32) wait_selftest(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival expected; none comes
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncwarp();
  mbar_wait(&bar, 0, &abort_flag, &g_tc_error, kErrWait, limit_ns);
}

// ============================================================== host side

// Dynamic shared memory of layer_tc<mode, kPh>.
template <int kPh>
int layer_smem_bytes(int mode) {
  return mode == kNoRope ? LayerCfg<kNoRope, kPh>::kSmemBytes
                         : (mode == kRopeTable ? LayerCfg<kRopeTable, kPh>::kSmemBytes
                                               : LayerCfg<kRopeOnTheFly, kPh>::kSmemBytes);
}

// Launch of layer_tc with programmatic dependent launch (the prologue may
// overlap the previous kernel in the stream); for the fused layer either as a
// cooperative launch (its CTAs wait on each other, so all must be resident) or
// with clusters of `cluster_x` CTAs along x (each cluster is co-scheduled).
cudaError_t launch_layer(void (*kern)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, Problem,
                                      RopeTable, LayerArgs),
                         int smem_bytes, dim3 grid, cudaStream_t s, bool cooperative,
                         const CUtensorMap& mk,
                         const CUtensorMap& mv, const CUtensorMap& mq, const CUtensorMap& mo,
                         const Problem& p, const RopeTable& rt, const LayerArgs& a,
                         int cluster_x = 0) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreadsTc, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem_bytes);
  cfg.stream = s;
  if (cluster_x > 0) {
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = static_cast<unsigned>(cluster_x);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, mk, mv, mq, mo, p, rt, a);
  }
  // A cooperative launch that the runtime refuses with the programmatic
  // attribute is retried without it (the kernel's griddepcontrol
  // instructions are then no-ops); the outcome is remembered.
  static std::atomic<int> coop_pdl{1};
  for (int attempt = 0; attempt < 2; ++attempt) {
    const bool pdl = !cooperative || coop_pdl.load() != 0;
    cudaLaunchAttribute attr[2];
    int n = 0;
    if (pdl) {
      attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[n].val.programmaticStreamSerializationAllowed = 1;
      ++n;
    }
    if (cooperative) {
      attr[n].id = cudaLaunchAttributeCooperative;
      attr[n].val.cooperative = 1;
      ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, mk, mv, mq, mo, p, rt, a);
    if (e == cudaSuccess || !cooperative || !pdl || e == cudaErrorCooperativeLaunchTooLarge)
      return e;
    (void)cudaGetLastError();
    coop_pdl.store(0);
  }
  return cudaErrorUnknown;
}

using LayerKernel = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, Problem,
                             RopeTable, LayerArgs);

// Whether every cluster of the cluster layer's grid (splits CTAs each, one
// per SM) can be resident at once, asked once per (RoPE mode, splits, device).
// Clusters must fit inside one GPC, so this can be less than the SM count
// divided by the cluster size.
int g_cluster_fit[3][kMaxCluster + 1][kMaxDev];  // 0 unknown, else co-resident clusters (-1 none)
std::mutex g_cluster_mu;

bool cluster_layer_fits(const Problem& p, int mode, LayerKernel kern) {
  if (p.splits < 1 || p.splits > kMaxCluster) return false;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return false;
  const long long clusters = static_cast<long long>((p.H + kGroupHeads - 1) / kGroupHeads) * p.B;
  std::lock_guard<std::mutex> lk(g_cluster_mu);
  int& known = g_cluster_fit[mode][p.splits][dev];
  if (known == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.splits, 1, 1);
    cfg.blockDim = dim3(kThreadsTc, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(layer_smem_bytes<kClusterLayer>(mode));
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(p.splits);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    const cudaError_t e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
    if (e != cudaSuccess) {
      (void)cudaGetLastError();
      n = 0;
    }
    known = n > 0 ? n : -1;  // cached: the number of co-resident clusters
  }
  return known > 0 && clusters <= known;
}

template <int kPh>
LayerKernel pick_kernel(int mode) {
  return mode == kNoRope ? layer_tc<kNoRope, kPh>
                         : (mode == kRopeTable ? layer_tc<kRopeTable, kPh>
                                               : layer_tc<kRopeOnTheFly, kPh>);
}

// 128-token tiles per CTA when `ctas` CTAs share a head group's tiles.
int apply_tiles_per_cta(const Problem& p, int ctas) {
  const int ntiles = (p.N + kApT - 1) / kApT;
  return (ntiles + ctas - 1) / ctas;
}

}  // namespace

cudaError_t launch_reduce_tc(const Problem& p, const void* K, const void* V, float* partials,
                             unsigned* counters, const StateOut& out, cudaStream_t s) {
  CUtensorMap mk, mv;
  cudaError_t e;
  if ((e = make_map(&mk, K, p, kRedT)) != cudaSuccess) return e;
  if ((e = make_map(&mv, V, p, kRedT)) != cudaSuccess) return e;
  const RopeTable rt = rope_table_for(p);
  const int mode = rope_mode(rt);
  LayerKernel kern = pick_kernel<kReduceOnly>(mode);
  const int kBytes = layer_smem_bytes<kReduceOnly>(mode);
  if ((e = ensure_smem_attr(mode, reinterpret_cast<const void*>(kern), kBytes)) != cudaSuccess)
    return e;
  LayerArgs a = {};
  a.partials = partials;
  a.arrive = counters;
  a.out = out;
  const dim3 grid(p.splits, (p.H + kGroupHeads - 1) / kGroupHeads, p.B);
  e = launch_layer(kern, kBytes, grid, s, false, mk, mv, mk, mk, p, rt, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_chunk_states_tc(const Problem& p, const void* K, const void* V, float* states,
                                   int nchunks, cudaStream_t s) {
  if (p.io != LA_IO_BF16 || p.N <= 0) return cudaErrorNotSupported;
  CUtensorMap mk, mv;
  cudaError_t e;
  if ((e = make_map(&mk, K, p, kRedT)) != cudaSuccess) return e;
  if ((e = make_map(&mv, V, p, kRedT)) != cudaSuccess) return e;
  const RopeTable rt = rope_table_for(p);
  const int mode = rope_mode(rt);
  LayerKernel kern = mode == kNoRope      ? layer_tc<kNoRope, kChunkStates>
                     : mode == kRopeTable ? layer_tc<kRopeTable, kChunkStates>
                                          : layer_tc<kRopeOnTheFly, kChunkStates>;
  const int kBytes = mode == kNoRope      ? LayerCfg<kNoRope, kChunkStates>::kSmemBytes
                     : mode == kRopeTable ? LayerCfg<kRopeTable, kChunkStates>::kSmemBytes
                                          : LayerCfg<kRopeOnTheFly, kChunkStates>::kSmemBytes;
  if ((e = ensure_smem_attr(12 + mode, reinterpret_cast<const void*>(kern), kBytes)) != cudaSuccess)
    return e;
  LayerArgs a = {};
  a.chunk_states = states;
  a.nchunks = nchunks;
  const dim3 grid(p.splits, (p.H + kGroupHeads - 1) / kGroupHeads, p.B);
  e = launch_layer(kern, kBytes, grid, s, false, mk, mv, mk, mk, p, rt, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_apply_tc(const Problem& p, const void* Q, const float* S, const float* z,
                            void* O, bool after_own_reduce, cudaStream_t s) {
  CUtensorMap mq, mo;
  cudaError_t e;
  if ((e = make_map(&mq, Q, p, kApT)) != cudaSuccess) return e;
  if ((e = make_map(&mo, O, p, kApT)) != cudaSuccess) return e;
  const RopeTable rt = rope_table_for(p);
  const int mode = rope_mode(rt);
  LayerKernel kern = pick_kernel<kApplyOnly>(mode);
  const int kBytes = layer_smem_bytes<kApplyOnly>(mode);
  if ((e = ensure_smem_attr(3 + mode, reinterpret_cast<const void*>(kern), kBytes)) !=
      cudaSuccess)
    return e;
  const int groups = (p.H + kGroupHeads - 1) / kGroupHeads;
  const int ntiles = (p.N + kApT - 1) / kApT;
  const long long units = static_cast<long long>(groups) * p.B;
  int ctas = static_cast<int>(std::max<long long>(1, kNumSMs / std::max<long long>(1, units)));
  ctas = std::min(ctas, ntiles);
  const int tpc = apply_tiles_per_cta(p, ctas);
  ctas = (ntiles + tpc - 1) / tpc;
  LayerArgs a = {};
  a.S_in = S;
  a.z_in = z;
  a.tiles_per_cta = tpc;
  // Q may be read before the previous kernel completes only when that kernel
  // is this library's own state reduce, which does not write Q and itself
  // started reading only after everything before it had completed.
  a.q_before_wait = after_own_reduce ? 1 : 0;
  const dim3 grid(ctas, groups, p.B);
  e = launch_layer(kern, kBytes, grid, s, false, mq, mq, mq, mo, p, rt, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// The single-launch layer runs whenever its CTAs fit one co-resident wave: with
// every CTA summing the split partials itself into shared memory, it measured
// faster than reduce + apply with programmatic dependent launch at every size
// here (1024px 22.6 vs 23.7 us, 4K 61.3 vs 62.6 us, video 118.4 vs 123.8 us).
// Both paths give bitwise identical results (same split order, same combine,
// same apply).
bool layer_fusable(const Problem& p) {
  const long long ctas =
      static_cast<long long>(p.splits) * ((p.H + kGroupHeads - 1) / kGroupHeads) * p.B;
  return p.io == LA_IO_BF16 && p.N > 0 && ctas <= kNumSMs;
}

cudaError_t launch_layer_tc(const Problem& p, const void* Q, const void* K, const void* V,
                            void* O, float* partials, unsigned* counters, const StateOut& out,
                            cudaStream_t s) {
  if (!layer_fusable(p) || out.out1_S == nullptr || out.out1_z == nullptr)
    return cudaErrorNotSupported;
  CUtensorMap mk, mv, mq, mo;
  cudaError_t e;
  if ((e = make_map(&mk, K, p, kRedT)) != cudaSuccess) return e;
  if ((e = make_map(&mv, V, p, kRedT)) != cudaSuccess) return e;
  if ((e = make_map(&mq, Q, p, kApT)) != cudaSuccess) return e;
  if ((e = make_map(&mo, O, p, kApT)) != cudaSuccess) return e;
  const RopeTable rt = rope_table_for(p);
  const int mode = rope_mode(rt);
  LayerKernel kern_cl = pick_kernel<kClusterLayer>(mode);
  const int kBytesCl = layer_smem_bytes<kClusterLayer>(mode);
  if ((e = ensure_smem_attr(9 + mode, reinterpret_cast<const void*>(kern_cl), kBytesCl)) !=
      cudaSuccess)
    return e;
  const dim3 grid(p.splits, (p.H + kGroupHeads - 1) / kGroupHeads, p.B);
  if (cluster_layer_fits(p, mode, kern_cl)) {
    // the head group's splits as one cluster: the hand-off stays on chip
    LayerArgs a = {};
    a.out = out;
    a.tiles_per_cta = apply_tiles_per_cta(p, p.splits);
    e = launch_layer(kern_cl, kBytesCl, grid, s, false, mk, mv, mq, mo, p, rt, a, p.splits);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  LayerKernel kern = pick_kernel<kFusedLayer>(mode);
  const int kBytes = layer_smem_bytes<kFusedLayer>(mode);
  if ((e = ensure_smem_attr(6 + mode, reinterpret_cast<const void*>(kern), kBytes)) !=
      cudaSuccess)
    return e;
  const size_t bh = static_cast<size_t>(p.B) * p.H;
  LayerArgs a = {};
  a.partials = partials;
  a.arrive = counters;
  a.ready = counters + bh;
  a.depart = counters + 2 * bh;
  a.out = out;
  a.S_in = out.out1_S;
  a.z_in = out.out1_z;
  a.tiles_per_cta = apply_tiles_per_cta(p, p.splits);
  e = launch_layer(kern, kBytes, grid, s, true, mk, mv, mq, mo, p, rt, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_wait_selftest(unsigned limit_us, cudaStream_t s) {
  wait_selftest<<<1, 32, 0, s>>>(static_cast<unsigned long long>(limit_us) * 1000ull);
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
