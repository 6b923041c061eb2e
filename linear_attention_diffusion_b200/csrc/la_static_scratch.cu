// la_state_reduce_static: the state reduce for callers that cannot hand the
// library a workspace.
//
// Some callers have no way to allocate device memory at the point where they
// run the reduce: a plugin inside a host application that owns every device
// buffer, a fixed-footprint runtime that forbids allocation once it has
// started, or a latency-critical loop that must not call cudaMalloc (which
// can synchronise the whole device). This entry point lets them run the
// reduce with only their inputs and outputs: its scratch (the per-split
// partial states and the per-head arrival counters) lives in a fixed array in
// the library's own device memory, declared below.
//
// Cost of that choice: every GPU that loads the library holds the array
// (kStaticScratchBytes) until the process exits, and all calls on one GPU
// share it. Calls whose kernels may run at the same time on one GPU (other
// streams, other host threads) race on the array and must be ordered by the
// caller.
#include <cuda.h>

#include "la_internal.h"
#include "la_scratch_cache.h"

namespace la {
namespace {

// 8 MiB. The scratch of a shape is a 256-aligned block of B*H arrival
// counters followed by B*H*splits partial states of (32*32 + 32) floats. The
// split rule gives one split per head group whenever B*ceil(H/4) > 74, and
// more splits only for smaller shapes (B*H <= 296), so a shape fits exactly
// when B*H <= 1984. The bench workloads need 2.4 MB: 70 heads x 8 splits for
// the 4K and video layers (B = 1), 4 x 70 heads x 2 splits for the 1024px
// layer.
constexpr size_t kStaticScratchBytes = size_t(8) << 20;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
SymbolAddressCache<kMaxDevices> g_scratch_cache;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
std::once_flag g_ctx_fn_once;
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;

bool load_ctx_functions() {
  std::call_once(g_ctx_fn_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(fn);
  });
  return g_ctx_get_current != nullptr && g_ctx_get_id != nullptr;
}

// Unique id of the context current on this thread; 0 when there is none yet.
cudaError_t current_context_id(unsigned long long* id) {
  *id = 0;
  CUcontext ctx = nullptr;
  if (g_ctx_get_current(&ctx) != CUDA_SUCCESS) return cudaErrorUnknown;
  if (ctx == nullptr) return cudaSuccess;
  return g_ctx_get_id(ctx, id) == CUDA_SUCCESS ? cudaSuccess : cudaErrorUnknown;
}

// Device address of g_static_scratch in the current device's context. In
// host code the array's name only stands for the symbol; the address a kernel
// may use comes from cudaGetSymbolAddress, called with the device current.
// The result is cached per device and keyed on the context id, so a context
// that was destroyed and created again (its module reloaded, the array
// possibly elsewhere) gets a fresh lookup instead of a stale address.
la_status scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return detail::cuda_fail(e, "la_state_reduce_static: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices)
    return detail::fail(LA_ERR_UNSUPPORTED, "la_state_reduce_static: device %d", dev);
  if (!load_ctx_functions())
    return detail::fail(LA_ERR_CUDA, "la_state_reduce_static: cuCtxGetCurrent / cuCtxGetId "
                                     "not available from the driver");
  unsigned long long ctx_id = 0;
  if ((e = current_context_id(&ctx_id)) != cudaSuccess)
    return detail::cuda_fail(e, "la_state_reduce_static: current context");
  if (ctx_id == 0) {
    // No context is current on this thread yet: the symbol lookup creates
    // the device's primary context and makes it current; key on that one.
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_static_scratch);
    if (e != cudaSuccess) return detail::cuda_fail(e, "la_state_reduce_static: cudaGetSymbolAddress");
    if ((e = current_context_id(&ctx_id)) != cudaSuccess || ctx_id == 0)
      return detail::cuda_fail(e == cudaSuccess ? cudaErrorDeviceUninitialized : e,
                               "la_state_reduce_static: current context");
  }
  cudaError_t lookup = cudaSuccess;
  const int rc = g_scratch_cache.get(dev, ctx_id, [&lookup](void** addr) {
    lookup = cudaGetSymbolAddress(addr, g_static_scratch);
    return (lookup == cudaSuccess && *addr != nullptr) ? 0 : 1;
  }, out);
  if (rc != 0)
    return detail::cuda_fail(lookup == cudaSuccess ? cudaErrorInvalidSymbol : lookup,
                             "la_state_reduce_static: cudaGetSymbolAddress");
  return LA_OK;
}

}  // namespace
}  // namespace la

using namespace la;

extern "C" la_status la_state_reduce_static(const la_shape* shape, const void* K, const void* V,
                                            float* S, float* z, la_stream stream) {
  Problem p;
  la_status st = detail::make_problem(shape, p);
  if (st != LA_OK) return st;
  const bool any_state = p.B > 0 && p.H > 0;
  const bool any_input = any_state && p.N > 0;
  if ((st = detail::check_ptr(K, "K", any_input)) != LA_OK) return st;
  if ((st = detail::check_ptr(V, "V", any_input)) != LA_OK) return st;
  if ((st = detail::check_ptr(S, "S", any_state)) != LA_OK) return st;
  if ((st = detail::check_ptr(z, "z", any_state)) != LA_OK) return st;
  const size_t bh = static_cast<size_t>(p.B) * p.H;
  if (detail::overlap(S, bh * kD * kD * 4, z, bh * kD * 4))
    return detail::fail(LA_ERR_INVALID_ARG, "S and z must not overlap");
  // Scratch layout: counters first, then the split partials.
  const size_t counters_bytes = detail::align256(bh * sizeof(unsigned));
  const size_t need = counters_bytes + bh * p.splits * kStateFloats * sizeof(float);
  if (need > kStaticScratchBytes)
    return detail::fail(LA_ERR_UNSUPPORTED,
                        "la_state_reduce_static: this shape needs %zu bytes of scratch but the "
                        "library's static array holds %zu; use la_state_reduce with a workspace",
                        need, kStaticScratchBytes);
  if (!any_state) return LA_OK;
  void* base = nullptr;
  if ((st = scratch_address(&base)) != LA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned char* scratch = static_cast<unsigned char*>(base);
  // The counters must start at zero; the array keeps whatever the previous
  // call (or a failed one) left there.
  cudaError_t e = cudaMemsetAsync(scratch, 0, bh * sizeof(unsigned), s);
  if (e != cudaSuccess) return detail::cuda_fail(e, "la_state_reduce_static: clear counters");
  const StateOut out = {nullptr, nullptr, S, z, nullptr, nullptr};
  e = launch_reduce(p, K, V, reinterpret_cast<float*>(scratch + counters_bytes),
                    reinterpret_cast<unsigned*>(scratch), out, s);
  if (e != cudaSuccess) return detail::cuda_fail(e, "la_state_reduce_static");
  return LA_OK;
}
