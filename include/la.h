/*
 * la.h -- C ABI of the B200 (sm_100a) ReLU linear-attention library.
 *
 * What the library computes, per batch element b and head h, with head
 * width D = 32 and eps >= 0:
 *
 *   k+ = ReLU(k),  q+ = ReLU(q)
 *   phi(x) = ReLU(x)                     (rope = 0)
 *   phi(x) = R(t, h, w) ReLU(x)          (rope = 1: 3D RoPE after ReLU)
 *   S = sum_n phi(k_n)^T v_n             (D x D, float32)
 *   z = sum_n k+_n                       (D, float32; never rotated)
 *   O_n = phi(q_n) S / (q+_n . z + eps)
 *
 * Sources (page title, section):
 *   "Sana: Efficient High-Resolution Image Synthesis with Linear Diffusion
 *   Transformers", section 模型架构 item 2: ReLU linear attention whose shared
 *   terms sum ReLU(K_j)^T V_j and sum ReLU(K_j)^T are computed once and reused
 *   by every query.
 *   "SANA-Video: Efficient Video Generation with Block Linear Diffusion
 *   Transformer", section 2.1 (state computed in advance, O(D^2) per token),
 *   section 2.2 (RoPE after ReLU; the denominator stays unrotated), section
 *   2.3 (causal state kept in D x D + D memory), section 4 (block inference
 *   loop: the KV cache starts empty and folds in each block once, after its
 *   last denoising step), "Stage 2" (3D RoPE over time, height and width).
 *
 * The formula of section 2.1 is lost on the pages. This library reads it as
 * above: no 1/sqrt(D) scale and eps added to the denominator.
 *
 * 3D RoPE convention (not fixed by the pages): dims [0,8) turn with the frame
 * index t, [8,20) with the row h, [20,32) with the column w; pairs (2i, 2i+1)
 * are interleaved; pair k of a segment of width d turns by
 * p * rope_base^(-2k/d); (x0, x1) -> (x0 cos - x1 sin, x0 sin + x1 cos).
 * Tokens are in raster order n = (t_local*Hh + h)*W + w and
 * t = t_offset + t_local is the global frame index.
 *
 * Conventions shared by every entry point:
 *   - Layout: Q, K, V, O are dense row-major [B, N, H, D] tensors of
 *     io_dtype (bf16 or float32). S is float32 [B, H, D, D] (row d, column
 *     e) and z is float32 [B, H, D].
 *   - Memory: every tensor pointer is a DEVICE pointer owned by the caller,
 *     16-byte aligned. The library allocates nothing and keeps no state
 *     between calls, with one exception: la_state_reduce_static keeps its
 *     scratch in a fixed 8 MiB device array that the library holds on every
 *     GPU it is loaded on (plus a host-side cache of that array's address per
 *     device and context); its calls on one GPU share the array and must be
 *     ordered when they could overlap. Scratch memory ("workspace") for
 *     every other entry point is passed in by the
 *     caller; its size comes from la_workspace_bytes(). A workspace must be
 *     zero-filled once before its first use (cudaMemsetAsync(ws, 0, bytes));
 *     every call leaves it zero-filled where it matters again, so it is
 *     reused without clearing. One workspace serves one call at a time:
 *     calls that share a workspace must be ordered (same stream or events).
 *     After a call that failed with LA_ERR_CUDA, zero-fill it again.
 *   - Execution: every call is asynchronous on `stream` (NULL = the legacy
 *     default stream). A call returns after enqueuing its kernels; faults
 *     inside kernels surface at the caller's next synchronisation.
 *   - Errors: arguments are checked on the host before any launch; a bad
 *     argument returns LA_ERR_INVALID_ARG / LA_ERR_UNSUPPORTED /
 *     LA_ERR_WORKSPACE and launches nothing. A launch failure returns
 *     LA_ERR_CUDA. Nothing throws across the ABI. la_last_error() gives a
 *     one-line description of the last failure on the calling thread.
 *   - Determinism: for a given shape the reduction order is fixed (split
 *     count and combine order depend on the shape only), so S, z and O are
 *     bitwise identical from run to run.
 *   - Aliasing: O must not overlap Q, K or V; S and z must not overlap the
 *     inputs or the workspace.
 */
#ifndef LA_H_
#define LA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so that this header needs no
 * CUDA header. */
typedef struct CUstream_st* la_stream;

typedef enum {
  LA_OK = 0,
  LA_ERR_INVALID_ARG = 1, /* null / misaligned pointer, negative size, bad flag */
  LA_ERR_UNSUPPORTED = 2, /* a valid request this build does not handle (D != 32) */
  LA_ERR_WORKSPACE = 3,   /* workspace missing or smaller than la_workspace_bytes() */
  LA_ERR_CUDA = 4         /* a CUDA runtime call or kernel launch failed */
} la_status;

typedef enum { LA_IO_BF16 = 0, LA_IO_F32 = 1 } la_io_dtype;

typedef struct {
  int B;            /* batch elements, >= 0 */
  int N;            /* tokens per batch element (per block in block-causal mode), >= 0 */
  int H;            /* heads, >= 0 */
  int D;            /* head width; must be 32 */
  int io_dtype;     /* la_io_dtype of Q, K, V and O */
  int rope;         /* 0: phi = ReLU; 1: phi = 3D RoPE after ReLU */
  int T, Hh, W;     /* RoPE latent grid; N == T*Hh*W when rope = 1 */
  int t_offset;     /* global frame index of this block's first frame, >= 0 */
  double rope_base; /* RoPE base (10000), > 1 */
  float eps;        /* denominator guard, >= 0 and finite */
} la_shape;

/* Bytes of scratch memory that la_state_reduce, la_attention and
 * la_block_causal_step need for `shape`. Returns 0 iff `shape` is invalid.
 * Pure host function; it does not touch the GPU. */
size_t la_workspace_bytes(const la_shape* shape);

/* State reduce (the shared terms of the Sana Linear DiT, section 模型架构
 * item 2; SANA-Video section 2.1):
 *   S[b,h] = sum_n phi(k_n)^T v_n,  z[b,h] = sum_n ReLU(k_n).
 * K, V: [B,N,H,D] io_dtype (device, read only). S: [B,H,D,D] float32, z:
 * [B,H,D] float32 (device, written). ws: device workspace of at least
 * la_workspace_bytes(shape) bytes (see the workspace rule above).
 * One launch: the token axis is cut into splits that depend on the shape
 * only; each CTA writes its split's partial state to the workspace and the
 * last CTA to finish for a head sums the partials in split order.
 * N == 0 gives S = 0, z = 0. */
la_status la_state_reduce(const la_shape* shape, const void* K, const void* V,
                          float* S, float* z, void* ws, size_t ws_bytes,
                          la_stream stream);

/* Apply (SANA-Video sections 2.1 and 2.2):
 *   O_n = phi(q_n) S / (ReLU(q_n) . z + eps).
 * Q: [B,N,H,D] io_dtype (read), S: [B,H,D,D] float32 and z: [B,H,D] float32
 * (read), O: [B,N,H,D] io_dtype (written; bf16 output is rounded to
 * nearest-even). A row with ReLU(q) = 0 gives O = 0. Needs no workspace. */
la_status la_apply(const la_shape* shape, const void* Q, const float* S,
                   const float* z, void* O, la_stream stream);

/* Non-causal attention in one call: la_state_reduce followed by la_apply.
 * S and z receive the state (they may be NULL, in which case the state is
 * kept in the workspace only). */
la_status la_attention(const la_shape* shape, const void* Q, const void* K,
                       const void* V, float* S, float* z, void* O, void* ws,
                       size_t ws_bytes, la_stream stream);

/* One call of the block-causal mode with the constant-memory KV cache
 * (SANA-Video sections 2.3 and 4; SANA-Video article, section 设计细节):
 * the block's own state (S_own, z_own) is reduced from (K, V), then
 *   update = 0: O = apply(Q, S_carry + S_own, z_carry + z_own); carry unchanged.
 *   update = 1: the same O; then S_carry += S_own, z_carry += z_own.
 *   update = 2: the carry update only; Q and O are not used (may be NULL).
 * Earlier blocks reach this block only through the carry; attention within
 * the block is global. S_carry [B,H,D,D], z_carry [B,H,D] float32 (device,
 * read and, for update >= 1, written in place). shape->t_offset is the global
 * frame index of the block's first frame. The sum carry + own is formed once,
 * in a fixed order, and the apply uses exactly the value stored in the carry
 * for update = 1. */
la_status la_block_causal_step(const la_shape* shape, const void* Q,
                               const void* K, const void* V, float* S_carry,
                               float* z_carry, void* O, int update, void* ws,
                               size_t ws_bytes, la_stream stream);

/* Backward of la_attention, for training (Sana, section Infra: the linear
 * attention is trained with a fused forward and backward kernel). Given the
 * forward's inputs, its state (S, z) and the output gradient dO, with
 * den_n = ReLU(q_n) . z + eps:
 *   dnum_n = dO_n / den_n,  dden_n = -(dO_n . O_n) / den_n,
 *   dS = sum_n phi(q_n)^T dnum_n,  dz = sum_n dden_n ReLU(q_n),
 *   dq_n = [R_n^T (S dnum_n^T) + dden_n z] * [q_n > 0],
 *   dk_n = [R_n^T (dS v_n^T) + dz] * [k_n > 0],  dv_n = phi(k_n) dS,
 * R_n the token's RoPE rotation (identity when shape->rope == 0), [x > 0]
 * taken elementwise (the gradient of ReLU at 0 is taken as 0).
 * Q, K, V, dO: [B,N,H,D] io_dtype (device, read). S [B,H,D,D], z [B,H,D]
 * float32 (device, read): the state the forward produced; both NULL makes the
 * call reduce it again from (K, V) into the workspace first. dQ, dK, dV:
 * [B,N,H,D] io_dtype (device, written; bf16 rounded to nearest-even).
 * dS [B,H,D,D], dz [B,H,D] float32 (device, written): the gradients of the
 * state. O is not an input: dO_n . O_n = phi(q_n) . (S dnum_n^T) / den_n.
 * ws: as for la_attention (same size). Two launches (three when the state is
 * recomputed); dS and dz are summed over the same shape-only token splits
 * as the state reduce, so results are bitwise reproducible.
 * None of the outputs may overlap each other, an input or the workspace. */
la_status la_attention_backward(const la_shape* shape, const void* Q,
                                const void* K, const void* V, const float* S,
                                const float* z, const void* dO, void* dQ,
                                void* dK, void* dV, float* dS, float* dz,
                                void* ws, size_t ws_bytes, la_stream stream);

/* Token-causal attention: query n sees keys 0..n (SANA-Video section 2.3
 * read at token granularity; the block-causal mode with blocks of one token).
 * With the carried state (S0, z0) = (S_carry, z_carry), or zero when both
 * are NULL:
 *   S_n = S0 + sum_{j<=n} phi(k_j)^T v_j,   z_n = z0 + sum_{j<=n} ReLU(k_j),
 *   O_n = phi(q_n) S_n / (ReLU(q_n) . z_n + eps).
 * update = 1 (needs the carry): afterwards the carry holds S_N, z_N, so a
 * sequence can be fed in consecutive calls (prefill, then one token at a
 * time); update = 0 leaves it unchanged. Q, K, V: [B,N,H,D] io_dtype (read);
 * O: [B,N,H,D] io_dtype (written); carry [B,H,D,D] / [B,H,D] float32. ws:
 * device workspace of at least la_causal_workspace_bytes(shape) bytes,
 * zero-filled once before its first use like the others.
 * bf16 I/O: three launches on the tensor cores (four with RoPE). The state
 * reduce writes every 128-token chunk's own state to the workspace (with RoPE
 * a second kernel adds the chunks' key sums of the unrotated ReLU(k)), a
 * prefix pass turns each into its chunk's exclusive prefix (the carry plus
 * the earlier chunks, summed in chunk order; update = 1 also folds the
 * sequence into the carry), and the output kernel computes every chunk
 * independently: the masked chunk-local product plus the chunk's prefix, the
 * weights and the rotated features carried in two bf16 parts each.
 * float32 I/O: two launches. The state reduce leaves each token split's
 * partial state in the workspace; a CUDA-core kernel starts each split from
 * the carry plus the earlier splits (summed in split order) and walks its
 * tokens in 32-token chunks. Deterministic either way. */
/* Bytes of workspace la_causal_attention needs for `shape` (at least
 * la_workspace_bytes(shape); for bf16, room for the state of every 128-token
 * chunk: B*H*ceil(N/128)*4224 bytes). 0 iff the shape is invalid. Pure host
 * function. */
size_t la_causal_workspace_bytes(const la_shape* shape);

la_status la_causal_attention(const la_shape* shape, const void* Q,
                              const void* K, const void* V, float* S_carry,
                              float* z_carry, void* O, int update, void* ws,
                              size_t ws_bytes, la_stream stream);

/* Shape of a channels-last video feature map [B][T][Hh][W][C] (the DiT's
 * tokens [B][N][C] with N = T*Hh*W in raster order). C must be a multiple
 * of 8. */
typedef struct {
  int B, T, Hh, W, C;
  int io_dtype; /* LA_IO_BF16 or LA_IO_F32 */
} la_conv_shape;

/* Temporal depth-wise convolution of the spatial-temporal Mix-FFN, entered
 * through a shortcut, with the block-causal conv cache f (SANA-Video, Stage 2
 * and section 4: the conv cache is the last frame of the temporal
 * convolution, the third part of the KV cache):
 *   y[t] = x[t] + bias + w[c][0] x[t-1] + w[c][1] x[t] + w[c][2] x[t+1]
 * per channel c, with x[-1] = f_in (the previous block's last frame; zero
 * when f_in is NULL, as for a whole clip or a first block) and x[T] = 0
 * (later blocks are never seen). f_out (may be NULL) receives x[T-1], the
 * cache for the next block. x, y: [B][T][Hh][W][C] io_dtype; f_in, f_out:
 * [B][Hh][W][C] io_dtype; w: [C][3] float32; bias: [C] float32 or NULL. All
 * device pointers, 16-byte aligned. y may be x (in place) and f_out may be
 * f_in; no other overlap is allowed. Float32 arithmetic, one rounding of y.
 * T = 0 leaves y empty and sets f_out to f_in (or zero). One launch. */
la_status la_temporal_conv(const la_conv_shape* shape, const void* x,
                           const float* w, const float* bias, const void* f_in,
                           void* f_out, void* y, la_stream stream);

/* Bytes of workspace la_qkv_state needs for `shape` and hidden width C.
 * Returns 0 iff the request is invalid or unsupported. Pure host function. */
size_t la_qkv_workspace_bytes(const la_shape* shape, int C);

/* QKV projection fused with the state reduce (Sana, section Infra: the
 * deployment GEMM of the QKV projection also forms ReLU(K)^T V, so the keys
 * and values never go to memory). For every token n of batch element b:
 *   [q_n, k_n, v_n] = bf16(W x_n + bias)    (float32 sum, one rounding each)
 * and then, exactly as la_state_reduce over those k and v:
 *   S[b,h] = sum_n phi(k_n)^T v_n,  z[b,h] = sum_n ReLU(k_n).
 * X: [B,N,C] bf16 token features (device, read). W: [3*H*D, C] bf16 (device,
 * read): rows [0, H*D) give the queries, [H*D, 2*H*D) the keys, [2*H*D,
 * 3*H*D) the values; head h owns rows [D*h, D*h + D) of each part. bias:
 * [3*H*D] bf16 in the same order, or NULL for none. Q: [B,N,H,D] bf16
 * (device, written): the queries. S [B,H,D,D], z [B,H,D] float32 (device,
 * written). shape->io_dtype must be LA_IO_BF16; rope, T, Hh, W and t_offset
 * select the feature map as for la_state_reduce (eps is not used). C: the
 * hidden width, a multiple of 8 in [8, 2^20]. ws: device workspace of at
 * least la_qkv_workspace_bytes(shape, C) bytes; it needs no zero fill.
 * Two launches: a persistent tensor-core GEMM that writes Q and one partial
 * state per run of key/value tiles, then a combine that sums each head's
 * partials in an order fixed by (B, N, H, C), so every bit of S and z is
 * reproducible. N == 0 gives S = 0, z = 0. Q, S and z must not overlap each
 * other, the inputs or the workspace. */
la_status la_qkv_state(const la_shape* shape, int C, const void* X,
                       const void* W, const void* bias, void* Q, float* S,
                       float* z, void* ws, size_t ws_bytes, la_stream stream);

/* Reset of the KV cache at the start of a video (SANA-Video section 4: the
 * cache starts empty): S[B,H,D,D] = 0, z[B,H,D] = 0 on `stream`. */
la_status la_state_reset(float* S, float* z, int B, int H, int D,
                         la_stream stream);

/* State reduce without a workspace, for callers that cannot allocate device
 * memory where they run it: a plugin inside a host application that owns
 * every device buffer, a fixed-footprint runtime that forbids allocation
 * after start-up, or a latency-critical loop that must not call cudaMalloc
 * (cudaMalloc can synchronise the device). The pages have no counterpart of
 * this entry point; it computes exactly what la_state_reduce computes, with
 * the same kernel and the same split order, so S and z are identical.
 *
 * Scratch: a fixed 8 MiB array in the library's own device memory. Every GPU
 * that loads the library holds it until the process exits. A shape whose
 * scratch (split partials + per-head counters) does not fit returns
 * LA_ERR_UNSUPPORTED before any launch; la_state_reduce with a workspace
 * handles it. The call allocates nothing and frees nothing; it clears the
 * counters it needs (cudaMemsetAsync on `stream`) before the kernel.
 * All calls on one GPU share the array: calls whose kernels may overlap on
 * the GPU (different streams or host threads) race and must be ordered.
 * The array's device address is looked up (cudaGetSymbolAddress) by the
 * first call in each CUDA context, with that context's device current, and
 * cached under the context's unique id, so a context created again after
 * cudaDeviceReset gets a fresh lookup; make the first call on each device
 * before any stream capture. */
la_status la_state_reduce_static(const la_shape* shape, const void* K,
                                 const void* V, float* S, float* z,
                                 la_stream stream);

/* Kernel launches that la_attention, and la_block_causal_step with update 0
 * or 1, make for `shape`: 1 when the whole layer runs as one cooperative
 * launch (bf16 I/O and a grid of splits x ceil(H/4) x B CTAs that fits one
 * wave of co-resident CTAs), else 2 (state reduce, then apply). The two give
 * bitwise identical results. 0 for an invalid shape. Pure host function. */
int la_attention_launches(const la_shape* shape);

/* Static description of a status code. Never NULL. */
const char* la_status_string(la_status status);

/* One-line description of the last failure on the calling thread (empty
 * string if none). The pointer stays valid until the thread's next call. */
const char* la_last_error(void);

/* Health check of the device-side waits: one warp waits for a barrier phase
 * that nothing completes; after limit_us microseconds (1 .. 10^7) it gives
 * up, raises bit 0 of the device error word (see la_device_error) and
 * returns, as a stalled pipeline stage of the library's kernels would. The
 * context stays usable. Asynchronous on `stream`; LA_OK means the launch
 * succeeded. */
la_status la_wait_selftest(unsigned limit_us, la_stream stream);

/* Device-side error word of the current device: non-zero when a kernel of
 * this library gave up on a bounded wait (a pipeline stage that never
 * arrived; the kernel then drained its copies and returned without a valid
 * result). Synchronous: waits for the device's pending work. `reset` != 0
 * clears the word afterwards. */
la_status la_device_error(unsigned* code, int reset);

#ifdef __cplusplus
}
#endif

#endif /* LA_H_ */
