// C-ABI layer: argument checks on the host, workspace layout, and the order
// of the kernel launches for each entry point of include/la.h.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "la.h"
#include "la_internal.h"

namespace la {
namespace detail {

thread_local std::string g_last_error;

la_status fail(la_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

la_status cuda_fail(cudaError_t e, const char* where) {
  return fail(LA_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Token splits of the state reduce: a function of (B, N, H) only, so that
// the reduction order, and with it every bit of S and z, is fixed per shape.
// One wave of CTAs of four heads (one CTA per SM), at least one 128-token
// tile per split.
void choose_splits(Problem& p) {
  const int groups = ceil_div(p.H, 4);
  const long long units = static_cast<long long>(p.B) * groups;
  int splits = units > 0 ? static_cast<int>(kNumSMs / units) : 1;
  const int max_splits = p.N > 0 ? ceil_div(p.N, kTileTokens) : 1;
  if (splits > max_splits) splits = max_splits;
  if (splits > 64) splits = 64;
  if (splits < 1) splits = 1;
  int chunk = p.N > 0 ? ceil_div(ceil_div(p.N, splits), kTileTokens) * kTileTokens : kTileTokens;
  p.chunk = chunk;
  p.splits = p.N > 0 ? ceil_div(p.N, chunk) : 1;
}

la_status make_problem(const la_shape* s, Problem& p) {
  if (s == nullptr) return fail(LA_ERR_INVALID_ARG, "shape is NULL");
  if (s->B < 0 || s->N < 0 || s->H < 0)
    return fail(LA_ERR_INVALID_ARG, "negative size B=%d N=%d H=%d", s->B, s->N, s->H);
  if (s->D != kD) return fail(LA_ERR_UNSUPPORTED, "head width D=%d (only 32 is built)", s->D);
  if (s->io_dtype != LA_IO_BF16 && s->io_dtype != LA_IO_F32)
    return fail(LA_ERR_INVALID_ARG, "io_dtype=%d", s->io_dtype);
  if (s->rope != 0 && s->rope != 1) return fail(LA_ERR_INVALID_ARG, "rope=%d", s->rope);
  if (!(std::isfinite(s->eps) && s->eps >= 0.0f))
    return fail(LA_ERR_INVALID_ARG, "eps must be finite and >= 0");
  const long long elems = 1LL * s->B * s->N * s->H * kD;
  if (elems >= (1LL << 40)) return fail(LA_ERR_UNSUPPORTED, "tensor too large");
  if (1LL * s->B * s->H * 65536LL >= (1LL << 40) || s->B > 65535 || s->H > 65535)
    return fail(LA_ERR_UNSUPPORTED, "B or H above 65535");
  std::memset(&p, 0, sizeof(p));
  p.B = s->B;
  p.N = s->N;
  p.H = s->H;
  p.io = s->io_dtype;
  p.eps = s->eps;
  if (s->rope) {
    if (s->T < 1 || s->Hh < 1 || s->W < 1)
      return fail(LA_ERR_INVALID_ARG, "RoPE grid T=%d Hh=%d W=%d", s->T, s->Hh, s->W);
    if (1LL * s->T * s->Hh * s->W != s->N)
      return fail(LA_ERR_INVALID_ARG, "N=%d != T*Hh*W=%lld", s->N, 1LL * s->T * s->Hh * s->W);
    if (s->t_offset < 0 || 1LL * s->t_offset + s->T > (1LL << 30))
      return fail(LA_ERR_INVALID_ARG, "t_offset=%d", s->t_offset);
    if (!(std::isfinite(s->rope_base) && s->rope_base > 1.0))
      return fail(LA_ERR_INVALID_ARG, "rope_base must be finite and > 1");
    p.rope.enabled = 1;
    p.rope.T = s->T;
    p.rope.Hh = s->Hh;
    p.rope.W = s->W;
    p.rope.t_offset = s->t_offset;
    // Segments of the head: 8 dims (4 pairs) time, 12 (6) height, 12 (6) width.
    const int seg_pairs[3] = {4, 6, 6};
    int j = 0;
    for (int a = 0; a < 3; ++a) {
      const int width = 2 * seg_pairs[a];
      for (int k = 0; k < seg_pairs[a]; ++k, ++j) {
        p.rope.axis[j] = a;
        p.rope.inv_freq[j] = std::pow(s->rope_base, -2.0 * k / width);
      }
    }
  }
  choose_splits(p);
  return LA_OK;
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

la_status check_ptr(const void* ptr, const char* name, bool needed) {
  if (!needed) return LA_OK;
  if (ptr == nullptr) return fail(LA_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned16(ptr)) return fail(LA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return LA_OK;
}

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (a == nullptr || b == nullptr || na == 0 || nb == 0) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

size_t io_bytes(const Problem& p) {
  return static_cast<size_t>(p.B) * p.N * p.H * kD * (p.io == 0 ? 2 : 4);
}
size_t s_bytes(const Problem& p) { return static_cast<size_t>(p.B) * p.H * kD * kD * 4; }
size_t z_bytes(const Problem& p) { return static_cast<size_t>(p.B) * p.H * kD * 4; }

#define LA_TRY(expr)                 \
  do {                               \
    const la_status st_ = (expr);    \
    if (st_ != LA_OK) return st_;    \
  } while (0)

la_status check_ws(const Problem& p, const void* ws, size_t ws_bytes) {
  const size_t need = workspace_layout(p).total;
  if (ws == nullptr) return fail(LA_ERR_WORKSPACE, "workspace is NULL (need %zu bytes)", need);
  if (!aligned16(ws)) return fail(LA_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
  if (ws_bytes < need)
    return fail(LA_ERR_WORKSPACE, "workspace of %zu bytes < %zu needed", ws_bytes, need);
  return LA_OK;
}

// Workspace of la_causal_attention: the chunk states of the chunked
// tensor-core path (bf16 without RoPE), else the ordinary layout.
size_t causal_workspace_bytes(const Problem& p) {
  const size_t base = workspace_layout(p).total;
  if (!causal_chunk_supported(p)) return base;
  return std::max(base, align256(causal_chunk_state_bytes(p)));
}

// State reduce of (K, V) into `out`, using the workspace's partials and
// counters.
la_status run_reduce(const Problem& p, const void* K, const void* V, char* ws,
                     const StateOut& out, cudaStream_t st) {
  const WsLayout L = workspace_layout(p);
  const cudaError_t e = launch_reduce(p, K, V, reinterpret_cast<float*>(ws + L.partials),
                                      reinterpret_cast<unsigned*>(ws + L.counters), out, st);
  if (e != cudaSuccess) return cuda_fail(e, "state reduce");
  return LA_OK;
}

}  // namespace detail

cudaError_t launch_reduce(const Problem& p, const void* K, const void* V, float* partials,
                          unsigned* counters, const StateOut& out, cudaStream_t s) {
  if (p.io == LA_IO_BF16 && p.N > 0) return launch_reduce_tc(p, K, V, partials, counters, out, s);
  return launch_reduce_simt(p, K, V, partials, counters, out, s);
}

cudaError_t launch_apply(const Problem& p, const void* Q, const float* S, const float* z,
                         void* O, bool after_own_reduce, cudaStream_t s) {
  if (p.io == LA_IO_BF16) return launch_apply_tc(p, Q, S, z, O, after_own_reduce && p.N > 0, s);
  return launch_apply_simt(p, Q, S, z, O, s);
}

cudaError_t launch_backward_q(const Problem& p, const void* Q, const void* dO, const float* S,
                              const float* z, void* dQ, float* partials, unsigned* counters,
                              const StateOut& out, cudaStream_t s) {
  if (p.io == LA_IO_BF16 && p.N > 0)
    return launch_backward_q_tc(p, Q, dO, S, z, dQ, partials, counters, out, s);
  return launch_backward_q_simt(p, Q, dO, S, z, dQ, partials, counters, out, s);
}

cudaError_t launch_backward_kv(const Problem& p, const void* K, const void* V, const float* dS,
                               const float* dz, void* dK, void* dV, bool after_own_q,
                               cudaStream_t s) {
  if (p.io == LA_IO_BF16) return launch_backward_kv_tc(p, K, V, dS, dz, dK, dV, after_own_q, s);
  return launch_backward_kv_simt(p, K, V, dS, dz, dK, dV, s);
}

WsLayout workspace_layout(const Problem& p) {
  using detail::align256;
  WsLayout L;
  const size_t bh = static_cast<size_t>(p.B) * p.H;
  L.counters = 0;
  L.partials = align256(3 * bh * sizeof(unsigned));
  L.state_S = align256(L.partials + bh * p.splits * kStateFloats * sizeof(float));
  L.state_z = align256(L.state_S + bh * kD * kD * sizeof(float));
  L.total = align256(L.state_z + bh * kD * sizeof(float));
  if (L.total == 0) L.total = 256;
  return L;
}

}  // namespace la

using namespace la;
using namespace la::detail;

extern "C" {

size_t la_causal_workspace_bytes(const la_shape* shape) {
  Problem p;
  if (make_problem(shape, p) != LA_OK) return 0;
  return causal_workspace_bytes(p);
}

size_t la_workspace_bytes(const la_shape* shape) {
  Problem p;
  if (make_problem(shape, p) != LA_OK) return 0;
  return workspace_layout(p).total;
}

la_status la_state_reduce(const la_shape* shape, const void* K, const void* V, float* S,
                          float* z, void* ws, size_t ws_bytes, la_stream stream) {
  Problem p;
  LA_TRY(make_problem(shape, p));
  const bool any_state = p.B > 0 && p.H > 0;
  const bool any_input = any_state && p.N > 0;
  LA_TRY(check_ptr(K, "K", any_input));
  LA_TRY(check_ptr(V, "V", any_input));
  LA_TRY(check_ptr(S, "S", any_state));
  LA_TRY(check_ptr(z, "z", any_state));
  LA_TRY(check_ws(p, ws, ws_bytes));
  if (overlap(S, s_bytes(p), ws, ws_bytes) || overlap(z, z_bytes(p), ws, ws_bytes) ||
      overlap(S, s_bytes(p), z, z_bytes(p)))
    return fail(LA_ERR_INVALID_ARG, "S, z and the workspace must not overlap");
  if (!any_state) return LA_OK;
  const StateOut out = {nullptr, nullptr, S, z, nullptr, nullptr};
  return run_reduce(p, K, V, static_cast<char*>(ws), out, reinterpret_cast<cudaStream_t>(stream));
}

la_status la_apply(const la_shape* shape, const void* Q, const float* S, const float* z,
                   void* O, la_stream stream) {
  Problem p;
  LA_TRY(make_problem(shape, p));
  const bool any = p.B > 0 && p.H > 0 && p.N > 0;
  LA_TRY(check_ptr(Q, "Q", any));
  LA_TRY(check_ptr(S, "S", any));
  LA_TRY(check_ptr(z, "z", any));
  LA_TRY(check_ptr(O, "O", any));
  if (overlap(O, io_bytes(p), Q, io_bytes(p)) || overlap(O, io_bytes(p), S, s_bytes(p)) ||
      overlap(O, io_bytes(p), z, z_bytes(p)))
    return fail(LA_ERR_INVALID_ARG, "O must not overlap Q, S or z");
  if (!any) return LA_OK;
  const cudaError_t e =
      launch_apply(p, Q, S, z, O, false, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "apply");
  return LA_OK;
}

la_status la_attention(const la_shape* shape, const void* Q, const void* K, const void* V,
                       float* S, float* z, void* O, void* ws, size_t ws_bytes,
                       la_stream stream) {
  Problem p;
  LA_TRY(make_problem(shape, p));
  const bool any_state = p.B > 0 && p.H > 0;
  const bool any_input = any_state && p.N > 0;
  LA_TRY(check_ptr(Q, "Q", any_input));
  LA_TRY(check_ptr(K, "K", any_input));
  LA_TRY(check_ptr(V, "V", any_input));
  LA_TRY(check_ptr(O, "O", any_input));
  if ((S == nullptr) != (z == nullptr))
    return fail(LA_ERR_INVALID_ARG, "S and z must both be given or both be NULL");
  LA_TRY(check_ptr(S, "S", any_state && S != nullptr));
  LA_TRY(check_ptr(z, "z", any_state && z != nullptr));
  LA_TRY(check_ws(p, ws, ws_bytes));
  const size_t nb = io_bytes(p);
  if (overlap(O, nb, Q, nb) || overlap(O, nb, K, nb) || overlap(O, nb, V, nb) ||
      overlap(O, nb, ws, ws_bytes) || overlap(S, s_bytes(p), ws, ws_bytes) ||
      overlap(z, z_bytes(p), ws, ws_bytes) || overlap(O, nb, S, s_bytes(p)) ||
      overlap(O, nb, z, z_bytes(p)))
    return fail(LA_ERR_INVALID_ARG, "O, S, z and the workspace must not overlap each other or the inputs");
  if (!any_state) return LA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  const WsLayout L = workspace_layout(p);
  float* Sw = reinterpret_cast<float*>(w + L.state_S);
  float* zw = reinterpret_cast<float*>(w + L.state_z);
  const StateOut out = {nullptr, nullptr, Sw, zw, S, z};
  if (any_input && layer_fusable(p)) {
    const cudaError_t e = launch_layer_tc(p, Q, K, V, O, reinterpret_cast<float*>(w + L.partials),
                                          reinterpret_cast<unsigned*>(w + L.counters), out, st);
    if (e == cudaSuccess) return LA_OK;
    if (e != cudaErrorNotSupported && e != cudaErrorCooperativeLaunchTooLarge)
      return cuda_fail(e, "attention layer");
    (void)cudaGetLastError();  // clear the refused launch, take the two-kernel path
  }
  LA_TRY(run_reduce(p, K, V, w, out, st));
  if (!any_input) return LA_OK;
  const cudaError_t e = launch_apply(p, Q, Sw, zw, O, true, st);
  if (e != cudaSuccess) return cuda_fail(e, "apply");
  return LA_OK;
}

la_status la_block_causal_step(const la_shape* shape, const void* Q, const void* K,
                               const void* V, float* S_carry, float* z_carry, void* O,
                               int update, void* ws, size_t ws_bytes, la_stream stream) {
  Problem p;
  LA_TRY(make_problem(shape, p));
  if (update < 0 || update > 2) return fail(LA_ERR_INVALID_ARG, "update=%d (0, 1 or 2)", update);
  const bool any_state = p.B > 0 && p.H > 0;
  const bool any_input = any_state && p.N > 0;
  const bool uses_q = update != 2;
  LA_TRY(check_ptr(Q, "Q", any_input && uses_q));
  LA_TRY(check_ptr(O, "O", any_input && uses_q));
  LA_TRY(check_ptr(K, "K", any_input));
  LA_TRY(check_ptr(V, "V", any_input));
  LA_TRY(check_ptr(S_carry, "S_carry", any_state));
  LA_TRY(check_ptr(z_carry, "z_carry", any_state));
  LA_TRY(check_ws(p, ws, ws_bytes));
  const size_t nb = io_bytes(p);
  if (overlap(S_carry, s_bytes(p), ws, ws_bytes) || overlap(z_carry, z_bytes(p), ws, ws_bytes) ||
      overlap(S_carry, s_bytes(p), z_carry, z_bytes(p)) ||
      (uses_q && (overlap(O, nb, Q, nb) || overlap(O, nb, K, nb) || overlap(O, nb, V, nb) ||
                  overlap(O, nb, ws, ws_bytes) || overlap(O, nb, S_carry, s_bytes(p)) ||
                  overlap(O, nb, z_carry, z_bytes(p)))))
    return fail(LA_ERR_INVALID_ARG, "O, the carry and the workspace must not overlap");
  if (!any_state) return LA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  const WsLayout L = workspace_layout(p);
  float* Sw = reinterpret_cast<float*>(w + L.state_S);
  float* zw = reinterpret_cast<float*>(w + L.state_z);
  // total = carry + own, formed once; written to the workspace for the apply
  // and, when updating, to the carry as well.
  const bool to_ws = uses_q;
  const bool to_carry = update >= 1;
  const StateOut out = {S_carry, z_carry, to_ws ? Sw : nullptr, to_ws ? zw : nullptr,
                        to_carry ? S_carry : nullptr, to_carry ? z_carry : nullptr};
  if (uses_q && any_input && layer_fusable(p)) {
    const cudaError_t e = launch_layer_tc(p, Q, K, V, O, reinterpret_cast<float*>(w + L.partials),
                                          reinterpret_cast<unsigned*>(w + L.counters), out, st);
    if (e == cudaSuccess) return LA_OK;
    if (e != cudaErrorNotSupported && e != cudaErrorCooperativeLaunchTooLarge)
      return cuda_fail(e, "block-causal layer");
    (void)cudaGetLastError();
  }
  LA_TRY(run_reduce(p, K, V, w, out, st));
  if (!uses_q || !any_input) return LA_OK;
  const cudaError_t e = launch_apply(p, Q, Sw, zw, O, true, st);
  if (e != cudaSuccess) return cuda_fail(e, "apply");
  return LA_OK;
}

la_status la_attention_backward(const la_shape* shape, const void* Q, const void* K,
                                const void* V, const float* S, const float* z, const void* dO,
                                void* dQ, void* dK, void* dV, float* dS, float* dz, void* ws,
                                size_t ws_bytes, la_stream stream) {
  Problem p;
  LA_TRY(make_problem(shape, p));
  const bool any_state = p.B > 0 && p.H > 0;
  const bool any_input = any_state && p.N > 0;
  if ((S == nullptr) != (z == nullptr))
    return fail(LA_ERR_INVALID_ARG, "S and z must both be given or both be NULL");
  const bool recompute = S == nullptr;
  LA_TRY(check_ptr(Q, "Q", any_input));
  LA_TRY(check_ptr(K, "K", any_input));
  LA_TRY(check_ptr(V, "V", any_input));
  LA_TRY(check_ptr(dO, "dO", any_input));
  LA_TRY(check_ptr(S, "S", any_state && !recompute));
  LA_TRY(check_ptr(z, "z", any_state && !recompute));
  LA_TRY(check_ptr(dQ, "dQ", any_input));
  LA_TRY(check_ptr(dK, "dK", any_input));
  LA_TRY(check_ptr(dV, "dV", any_input));
  LA_TRY(check_ptr(dS, "dS", any_state));
  LA_TRY(check_ptr(dz, "dz", any_state));
  LA_TRY(check_ws(p, ws, ws_bytes));
  const size_t nb = io_bytes(p), sb = s_bytes(p), zb = z_bytes(p);
  const void* outs[5] = {dQ, dK, dV, dS, dz};
  const size_t out_n[5] = {nb, nb, nb, sb, zb};
  const void* ins[7] = {Q, K, V, dO, S, z, ws};
  const size_t in_n[7] = {nb, nb, nb, nb, sb, zb, ws_bytes};
  for (int i = 0; i < 5; ++i) {
    for (int j = i + 1; j < 5; ++j)
      if (overlap(outs[i], out_n[i], outs[j], out_n[j]))
        return fail(LA_ERR_INVALID_ARG, "the gradients must not overlap each other");
    for (int j = 0; j < 7; ++j)
      if (overlap(outs[i], out_n[i], ins[j], in_n[j]))
        return fail(LA_ERR_INVALID_ARG, "a gradient overlaps an input or the workspace");
  }
  if (!recompute && (overlap(S, sb, ws, ws_bytes) || overlap(z, zb, ws, ws_bytes)))
    return fail(LA_ERR_INVALID_ARG, "S and z must not overlap the workspace");
  if (!any_state) return LA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  const WsLayout L = workspace_layout(p);
  float* partials = reinterpret_cast<float*>(w + L.partials);
  unsigned* counters = reinterpret_cast<unsigned*>(w + L.counters);
  if (recompute) {
    float* Sw = reinterpret_cast<float*>(w + L.state_S);
    float* zw = reinterpret_cast<float*>(w + L.state_z);
    LA_TRY(run_reduce(p, K, V, w, StateOut{nullptr, nullptr, Sw, zw, nullptr, nullptr}, st));
    S = Sw;
    z = zw;
  }
  const StateOut grads = {nullptr, nullptr, dS, dz, nullptr, nullptr};
  cudaError_t e = launch_backward_q(p, Q, dO, S, z, dQ, partials, counters, grads, st);
  if (e != cudaSuccess) return cuda_fail(e, "backward (query side)");
  if (!any_input) return LA_OK;
  e = launch_backward_kv(p, K, V, dS, dz, dK, dV, true, st);
  if (e != cudaSuccess) return cuda_fail(e, "backward (key side)");
  return LA_OK;
}

la_status la_causal_attention(const la_shape* shape, const void* Q, const void* K,
                              const void* V, float* S_carry, float* z_carry, void* O, int update,
                              void* ws, size_t ws_bytes, la_stream stream) {
  Problem p;
  LA_TRY(make_problem(shape, p));
  if (update < 0 || update > 1) return fail(LA_ERR_INVALID_ARG, "update=%d (0 or 1)", update);
  if ((S_carry == nullptr) != (z_carry == nullptr))
    return fail(LA_ERR_INVALID_ARG, "S_carry and z_carry must both be given or both be NULL");
  if (update == 1 && S_carry == nullptr)
    return fail(LA_ERR_INVALID_ARG, "update=1 needs S_carry and z_carry");
  const bool any_state = p.B > 0 && p.H > 0;
  const bool any_input = any_state && p.N > 0;
  LA_TRY(check_ptr(Q, "Q", any_input));
  LA_TRY(check_ptr(K, "K", any_input));
  LA_TRY(check_ptr(V, "V", any_input));
  LA_TRY(check_ptr(O, "O", any_input));
  LA_TRY(check_ptr(S_carry, "S_carry", any_state && S_carry != nullptr));
  LA_TRY(check_ptr(z_carry, "z_carry", any_state && z_carry != nullptr));
  {
    const size_t need = causal_workspace_bytes(p);
    if (ws == nullptr) return fail(LA_ERR_WORKSPACE, "workspace is NULL (need %zu bytes)", need);
    if (!aligned16(ws)) return fail(LA_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
    if (ws_bytes < need)
      return fail(LA_ERR_WORKSPACE, "workspace of %zu bytes < %zu needed (la_causal_workspace_bytes)",
                  ws_bytes, need);
  }
  const size_t nb = io_bytes(p);
  if (overlap(O, nb, Q, nb) || overlap(O, nb, K, nb) || overlap(O, nb, V, nb) ||
      overlap(O, nb, ws, ws_bytes) || overlap(O, nb, S_carry, s_bytes(p)) ||
      overlap(O, nb, z_carry, z_bytes(p)) || overlap(S_carry, s_bytes(p), ws, ws_bytes) ||
      overlap(z_carry, z_bytes(p), ws, ws_bytes) ||
      overlap(S_carry, s_bytes(p), z_carry, z_bytes(p)))
    return fail(LA_ERR_INVALID_ARG, "O, the carry and the workspace must not overlap");
  if (!any_state) return LA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  if (causal_chunk_supported(p)) {
    // bf16: every chunk's state (and with RoPE its key sums), their prefix,
    // then the chunks
    const cudaError_t e = launch_causal_chunks(p, Q, K, V, reinterpret_cast<float*>(w), S_carry,
                                               z_carry, update, O, st);
    if (e != cudaSuccess) return cuda_fail(e, "causal attention");
    return LA_OK;
  }
  const WsLayout L = workspace_layout(p);
  // the splits' partial states only: no combine
  LA_TRY(run_reduce(p, K, V, w, StateOut{nullptr, nullptr, nullptr, nullptr, nullptr, nullptr},
                    st));
  const float* partials = reinterpret_cast<const float*>(w + L.partials);
  unsigned* counters = reinterpret_cast<unsigned*>(w + L.counters);
  const cudaError_t e =
      launch_causal(p, Q, K, V, partials, S_carry, z_carry, update, counters, O, st);
  if (e != cudaSuccess) return cuda_fail(e, "causal attention");
  return LA_OK;
}

la_status la_temporal_conv(const la_conv_shape* shape, const void* x, const float* w,
                           const float* bias, const void* f_in, void* f_out, void* y,
                           la_stream stream) {
  if (shape == nullptr) return fail(LA_ERR_INVALID_ARG, "shape is NULL");
  const la_conv_shape& s = *shape;
  if (s.B < 0 || s.T < 0 || s.Hh < 0 || s.W < 0 || s.C < 0)
    return fail(LA_ERR_INVALID_ARG, "negative size B=%d T=%d Hh=%d W=%d C=%d", s.B, s.T, s.Hh,
                s.W, s.C);
  if (s.C % 8 != 0) return fail(LA_ERR_UNSUPPORTED, "C=%d is not a multiple of 8", s.C);
  if (s.io_dtype != LA_IO_BF16 && s.io_dtype != LA_IO_F32)
    return fail(LA_ERR_INVALID_ARG, "io_dtype=%d", s.io_dtype);
  const long long hw = 1LL * s.Hh * s.W;
  const long long frame_elems = hw * s.C;
  if (hw > 0x7fffffffLL || 1LL * s.B * s.T * frame_elems >= (1LL << 40))
    return fail(LA_ERR_UNSUPPORTED, "feature map too large");
  const size_t esz = s.io_dtype == LA_IO_BF16 ? 2 : 4;
  const size_t nx = static_cast<size_t>(s.B) * s.T * frame_elems * esz;
  const size_t nf = static_cast<size_t>(s.B) * frame_elems * esz;
  const bool any_cols = s.B > 0 && hw > 0 && s.C > 0;
  const bool any = any_cols && s.T > 0;
  LA_TRY(check_ptr(x, "x", any));
  LA_TRY(check_ptr(y, "y", any));
  LA_TRY(check_ptr(w, "w", any));
  LA_TRY(check_ptr(bias, "bias", any && bias != nullptr));
  LA_TRY(check_ptr(f_in, "f_in", any_cols && f_in != nullptr));
  LA_TRY(check_ptr(f_out, "f_out", any_cols && f_out != nullptr));
  const size_t nw = static_cast<size_t>(s.C) * 3 * 4, nb = static_cast<size_t>(s.C) * 4;
  // y == x and f_out == f_in are allowed exactly; any other overlap is not
  if ((y != x && overlap(y, nx, x, nx)) || (f_out != f_in && overlap(f_out, nf, f_in, nf)) ||
      overlap(y, nx, w, nw) || overlap(y, nx, bias, nb) || overlap(y, nx, f_in, nf) ||
      overlap(y, nx, f_out, nf) || overlap(f_out, nf, x, nx) || overlap(f_out, nf, w, nw) ||
      overlap(f_out, nf, bias, nb))
    return fail(LA_ERR_INVALID_ARG, "y and f_out must not overlap the other buffers");
  if (!any_cols) return LA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (s.T == 0) {
    if (f_out == nullptr || f_out == f_in) return LA_OK;
    const cudaError_t e = f_in != nullptr
                              ? cudaMemcpyAsync(f_out, f_in, nf, cudaMemcpyDeviceToDevice, st)
                              : cudaMemsetAsync(f_out, 0, nf, st);
    if (e != cudaSuccess) return cuda_fail(e, "temporal conv (empty clip)");
    return LA_OK;
  }
  ConvProblem cp;
  cp.B = s.B;
  cp.T = s.T;
  cp.HW = static_cast<int>(hw);
  cp.C = s.C;
  cp.io = s.io_dtype;
  const cudaError_t e = launch_temporal_conv(cp, x, w, bias, f_in, f_out, y, st);
  if (e != cudaSuccess) return cuda_fail(e, "temporal conv");
  return LA_OK;
}

// Hidden width of la_qkv_state: at least 8, a multiple of 8 (rows of X and W
// are 16-byte aligned for TMA), and small enough for 32-bit tile arithmetic.
static la_status check_qkv(const la_shape* shape, int C, Problem& p) {
  LA_TRY(make_problem(shape, p));
  if (p.io != LA_IO_BF16)
    return fail(LA_ERR_UNSUPPORTED, "la_qkv_state takes bf16 tensors only (io_dtype=%d)", p.io);
  if (C < 8 || C % 8 != 0 || C > (1 << 20))
    return fail(LA_ERR_UNSUPPORTED, "hidden width C=%d (a multiple of 8 in [8, 2^20])", C);
  const long long tiles = 1LL * p.B * ((p.N + 127) / 128) * ((p.H + 3) / 4 + (p.H * kD + 255) / 256);
  if (tiles >= (1LL << 30)) return fail(LA_ERR_UNSUPPORTED, "projection too large");
  return LA_OK;
}

size_t la_qkv_workspace_bytes(const la_shape* shape, int C) {
  Problem p;
  if (check_qkv(shape, C, p) != LA_OK) return 0;
  const size_t n = align256(qkv_workspace_floats(p.B, p.N, p.H, C) * sizeof(float));
  return n == 0 ? 256 : n;
}

la_status la_qkv_state(const la_shape* shape, int C, const void* X, const void* W,
                       const void* bias, void* Q, float* S, float* z, void* ws, size_t ws_bytes,
                       la_stream stream) {
  Problem p;
  LA_TRY(check_qkv(shape, C, p));
  const bool any_state = p.B > 0 && p.H > 0;
  const bool any = any_state && p.N > 0;
  LA_TRY(check_ptr(X, "X", any));
  LA_TRY(check_ptr(W, "W", any));
  LA_TRY(check_ptr(bias, "bias", any && bias != nullptr));
  LA_TRY(check_ptr(Q, "Q", any));
  LA_TRY(check_ptr(S, "S", any_state));
  LA_TRY(check_ptr(z, "z", any_state));
  const size_t hd = static_cast<size_t>(p.H) * kD;
  const size_t nx = static_cast<size_t>(p.B) * p.N * C * 2, nw = 3 * hd * C * 2, nb = 3 * hd * 2;
  const size_t nq = static_cast<size_t>(p.B) * p.N * hd * 2;
  const size_t need = any ? la_qkv_workspace_bytes(shape, C) : 0;
  if (any) {
    if (ws == nullptr) return fail(LA_ERR_WORKSPACE, "workspace is NULL (need %zu bytes)", need);
    if (!aligned16(ws)) return fail(LA_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
    if (ws_bytes < need)
      return fail(LA_ERR_WORKSPACE, "workspace of %zu bytes < %zu needed", ws_bytes, need);
  }
  const size_t ns = s_bytes(p), nz = z_bytes(p);
  const void* ins[4] = {X, W, bias, ws};
  const size_t in_n[4] = {nx, nw, bias != nullptr ? nb : 0, need};
  void* outs[3] = {Q, S, z};
  const size_t out_n[3] = {any ? nq : 0, ns, nz};
  for (int a = 0; a < 3; ++a) {
    for (int b = 0; b < 4; ++b)
      if (overlap(outs[a], out_n[a], ins[b], in_n[b]))
        return fail(LA_ERR_INVALID_ARG, "Q, S and z must not overlap X, W, bias or the workspace");
    for (int b = a + 1; b < 3; ++b)
      if (overlap(outs[a], out_n[a], outs[b], out_n[b]))
        return fail(LA_ERR_INVALID_ARG, "Q, S and z must not overlap each other");
  }
  if (!any_state) return LA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (p.N == 0) {  // no tokens: the state of an empty sequence
    cudaError_t e = cudaMemsetAsync(S, 0, ns, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(z, 0, nz, st);
    if (e != cudaSuccess) return cuda_fail(e, "la_qkv_state (empty sequence)");
    return LA_OK;
  }
  const cudaError_t e =
      launch_qkv_state(p, C, X, W, bias, Q, S, z, static_cast<float*>(ws), st);
  if (e != cudaSuccess) return cuda_fail(e, "la_qkv_state");
  return LA_OK;
}

la_status la_state_reset(float* S, float* z, int B, int H, int D, la_stream stream) {
  if (B < 0 || H < 0) return fail(LA_ERR_INVALID_ARG, "negative size B=%d H=%d", B, H);
  if (D != kD) return fail(LA_ERR_UNSUPPORTED, "head width D=%d (only 32 is built)", D);
  const bool any = B > 0 && H > 0;
  LA_TRY(check_ptr(S, "S", any));
  LA_TRY(check_ptr(z, "z", any));
  if (!any) return LA_OK;
  const size_t bh = static_cast<size_t>(B) * H;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(S, 0, bh * kD * kD * sizeof(float), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(z, 0, bh * kD * sizeof(float), st);
  if (e != cudaSuccess) return cuda_fail(e, "state reset");
  return LA_OK;
}

int la_attention_launches(const la_shape* shape) {
  Problem p;
  if (make_problem(shape, p) != LA_OK) return 0;
  if (p.B == 0 || p.H == 0) return 0;
  if (p.N == 0) return 1;
  return layer_fusable(p) ? 1 : 2;
}

const char* la_status_string(la_status status) {
  switch (status) {
    case LA_OK: return "LA_OK";
    case LA_ERR_INVALID_ARG: return "LA_ERR_INVALID_ARG: invalid argument";
    case LA_ERR_UNSUPPORTED: return "LA_ERR_UNSUPPORTED: unsupported request";
    case LA_ERR_WORKSPACE: return "LA_ERR_WORKSPACE: workspace missing or too small";
    case LA_ERR_CUDA: return "LA_ERR_CUDA: CUDA runtime or launch failure";
  }
  return "unknown la_status";
}

const char* la_last_error(void) { return g_last_error.c_str(); }

la_status la_wait_selftest(unsigned limit_us, la_stream stream) {
  if (limit_us == 0 || limit_us > 10000000u)
    return fail(LA_ERR_INVALID_ARG, "limit_us=%u (1 .. 10^7)", limit_us);
  const cudaError_t e = launch_wait_selftest(limit_us, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "wait self-test");
  return LA_OK;
}

la_status la_device_error(unsigned* code, int reset) {
  if (code == nullptr) return fail(LA_ERR_INVALID_ARG, "code is NULL");
  unsigned fwd = 0, bwd = 0, conv = 0, causal = 0, qkv = 0;
  cudaError_t e = read_device_error(&fwd, reset != 0);
  if (e == cudaSuccess) e = read_device_error_bwd(&bwd, reset != 0);
  if (e == cudaSuccess) e = read_device_error_conv(&conv, reset != 0);
  if (e == cudaSuccess) e = read_device_error_causal_chunk(&causal, reset != 0);
  if (e == cudaSuccess) e = read_device_error_qkv(&qkv, reset != 0);
  if (e != cudaSuccess) return cuda_fail(e, "la_device_error");
  *code = fwd | bwd | conv | causal | qkv;
  return LA_OK;
}

}  // extern "C"
