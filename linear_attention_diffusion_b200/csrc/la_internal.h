// Internal interface between the C-ABI layer (la_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "la.h"

namespace la {

constexpr int kD = 32;                 // head width (the only one supported)
constexpr int kStateFloats = kD * kD + kD;  // one (S, z) pair: 32x32 + 32
constexpr int kNumSMs = 148;           // B200; used for the shape-only split rule
constexpr int kTileTokens = 128;       // token granularity of a split

// 3D RoPE: per pair j in [0,16) the axis (0 = t, 1 = h, 2 = w) and the inverse
// frequency base^(-2k/d) of its segment, computed on the host in double.
struct Rope {
  int enabled;
  int T, Hh, W, t_offset;
  double inv_freq[kD / 2];
  int axis[kD / 2];
};

struct Problem {
  int B, N, H;
  int io;      // 0 bf16, 1 float32
  float eps;
  int splits;  // token splits of the state reduce (shape-only)
  int chunk;   // tokens per split (multiple of kTileTokens)
  Rope rope;
};

// Workspace layout (byte offsets, 256-aligned), a pure function of the shape.
struct WsLayout {
  size_t counters;  // [3][B*H] uint32 arrival / ready / departure words; zero between calls
  size_t partials;  // [B*H][splits][kStateFloats] float32
  size_t state_S;   // [B*H][32*32] float32
  size_t state_z;   // [B*H][32] float32
  size_t total;
};
WsLayout workspace_layout(const Problem& p);

// Where the reduce puts its result: the fixed-order sum of the split
// partials, plus carry_* when given, is written to out1_* and/or out2_*
// (each may be null; out2 may alias carry). All [B*H][32*32] / [B*H][32].
struct StateOut {
  const float* carry_S;
  const float* carry_z;
  float* out1_S;
  float* out1_z;
  float* out2_S;
  float* out2_z;
};

// State reduce in one launch: every CTA writes its split's partial (S, z)
// to `partials`; the last CTA to arrive for a head (counted in `counters`)
// sums the partials in split order, applies StateOut, and re-zeroes the
// counter. Deterministic: the sum order depends on the shape only.
cudaError_t launch_reduce(const Problem& p, const void* K, const void* V, float* partials,
                          unsigned* counters, const StateOut& out, cudaStream_t s);
// O = phi(Q) S / (ReLU(Q) . z + eps). after_own_reduce: the previous kernel
// on the stream is this library's state reduce (so Q may be read early).
cudaError_t launch_apply(const Problem& p, const void* Q, const float* S,
                         const float* z, void* O, bool after_own_reduce, cudaStream_t s);

// The two implementations behind launch_reduce / launch_apply: tensor-core
// kernels for bf16 I/O (la_tc.cu), CUDA-core kernels for float32 I/O and the
// empty sequence (la_simt.cu).
cudaError_t launch_reduce_tc(const Problem& p, const void* K, const void* V, float* partials,
                             unsigned* counters, const StateOut& out, cudaStream_t s);
cudaError_t launch_apply_tc(const Problem& p, const void* Q, const float* S, const float* z,
                            void* O, bool after_own_reduce, cudaStream_t s);
cudaError_t launch_reduce_simt(const Problem& p, const void* K, const void* V, float* partials,
                               unsigned* counters, const StateOut& out, cudaStream_t s);
cudaError_t launch_apply_simt(const Problem& p, const void* Q, const float* S, const float* z,
                              void* O, cudaStream_t s);
// The whole layer (state reduce, then apply) in one cooperative launch; the
// reduce's combined state goes to `out` (out.out1_* must be set: the apply
// reads it there). Returns cudaErrorNotSupported when the shape does not fit
// one wave of co-resident CTAs; the caller then launches reduce and apply.
bool layer_fusable(const Problem& p);
cudaError_t launch_layer_tc(const Problem& p, const void* Q, const void* K, const void* V,
                            void* O, float* partials, unsigned* counters, const StateOut& out,
                            cudaStream_t s);
// Backward of the non-causal layer. Query side: dQ, and the state gradients
// reduced over the token splits into `out` (same partials, counters and split
// order as the state reduce). Key side: dK and dV from the combined dS, dz.
// Tensor-core kernels for bf16 I/O (la_backward_tc.cu), CUDA-core kernels for
// float32 I/O and the empty sequence (la_backward.cu).
cudaError_t launch_backward_q(const Problem& p, const void* Q, const void* dO, const float* S,
                              const float* z, void* dQ, float* partials, unsigned* counters,
                              const StateOut& out, cudaStream_t s);
cudaError_t launch_backward_kv(const Problem& p, const void* K, const void* V, const float* dS,
                               const float* dz, void* dK, void* dV, bool after_own_q,
                               cudaStream_t s);
cudaError_t launch_backward_q_tc(const Problem& p, const void* Q, const void* dO, const float* S,
                                 const float* z, void* dQ, float* partials, unsigned* counters,
                                 const StateOut& out, cudaStream_t s);
cudaError_t launch_backward_kv_tc(const Problem& p, const void* K, const void* V, const float* dS,
                                  const float* dz, void* dK, void* dV, bool after_own_q,
                                  cudaStream_t s);
cudaError_t launch_backward_q_simt(const Problem& p, const void* Q, const void* dO,
                                   const float* S, const float* z, void* dQ, float* partials,
                                   unsigned* counters, const StateOut& out, cudaStream_t s);
cudaError_t launch_backward_kv_simt(const Problem& p, const void* K, const void* V,
                                    const float* dS, const float* dz, void* dK, void* dV,
                                    cudaStream_t s);
// Token-causal attention (la_causal.cu): `partials` holds every token
// split's partial state (the state reduce with no outputs requested); each
// split starts from the carry plus the earlier splits' partials. update = 1
// folds the whole sequence into the carry (read-before-write is ordered by
// `counters`, which the kernel leaves zero).
cudaError_t launch_causal(const Problem& p, const void* Q, const void* K, const void* V,
                          const float* partials, float* S_carry, float* z_carry, int update,
                          unsigned* counters, void* O, cudaStream_t s);
// The chunked tensor-core version (la_causal_chunk.cu, bf16 I/O without
// RoPE): the state reduce writes every 128-token chunk's own state into
// `states` (causal_chunk_state_bytes), a prefix kernel turns them into each
// chunk's exclusive prefix (carry included; update = 1 folds the sequence into
// the carry), and the output kernel computes every chunk independently.
bool causal_chunk_supported(const Problem& p);
size_t causal_chunk_state_bytes(const Problem& p);
cudaError_t launch_chunk_states_tc(const Problem& p, const void* K, const void* V, float* states,
                                   int nchunks, cudaStream_t s);
cudaError_t launch_causal_chunks(const Problem& p, const void* Q, const void* K, const void* V,
                                 float* states, float* S_carry, float* z_carry, int update,
                                 void* O, cudaStream_t s);
cudaError_t read_device_error_causal_chunk(unsigned* code, bool reset);
// Temporal depth-wise convolution with the conv cache (la_conv.cu).
struct ConvProblem {
  int B, T, HW, C;  // C a multiple of 8
  int io;           // 0 bf16, 1 float32
};
cudaError_t launch_temporal_conv(const ConvProblem& cp, const void* x, const float* w,
                                 const float* bias, const void* f_in, void* f_out, void* y,
                                 cudaStream_t s);
// Device error words of the tensor-core kernels (bounded waits that gave up):
// the forward's (la_tc.cu) and the backward's (la_backward_tc.cu).
cudaError_t read_device_error(unsigned* code, bool reset);
// One warp waiting on a barrier that nothing completes, bounded by limit_us.
cudaError_t launch_wait_selftest(unsigned limit_us, cudaStream_t s);
cudaError_t read_device_error_bwd(unsigned* code, bool reset);
cudaError_t read_device_error_conv(unsigned* code, bool reset);  // la_conv.cu
cudaError_t read_device_error_qkv(unsigned* code, bool reset);     // la_qkv_tc.cu
// QKV projection fused with the state reduce (la_qkv_tc.cu): a persistent
// tcgen05 GEMM that writes Q and one partial state per run of key/value
// tiles into `part` (qkv_workspace_floats floats), then a combine kernel that
// sums the partials in a fixed order into S and z. bf16 only, N > 0.
size_t qkv_workspace_floats(int B, int N, int H, int C);
cudaError_t launch_qkv_state(const Problem& p, int C, const void* X, const void* W,
                             const void* bias, void* Q, float* S, float* z, float* part,
                             cudaStream_t s);

// Host-side helpers of the C-ABI layer (la_api.cu).
namespace detail {
la_status fail(la_status st, const char* fmt, ...);
la_status cuda_fail(cudaError_t e, const char* where);
la_status make_problem(const la_shape* s, Problem& p);
la_status check_ptr(const void* ptr, const char* name, bool needed);
bool overlap(const void* a, size_t na, const void* b, size_t nb);
size_t align256(size_t x);
}  // namespace detail

}  // namespace la
