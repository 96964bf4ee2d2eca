/*
 * moe.h -- C ABI of the B200 (sm_100a) hard-routed sparse MoE layer forward.
 *
 * The layer, for T tokens x [T][d], E experts, top-k routing and expert
 * hidden size F (SwiGLU experts):
 *
 *   logits  L = x . W_r + b                                    (moe_route)
 *   top-k   idx[t][0..k-1], w[t][j] = softmax over the selected (moe_route / moe_topk)
 *   sort    routed slots r = t*k + j sorted by expert           (moe_sort_rows)
 *   gate|up h[i] = silu(x[row_map[i]] Wg_e^T) * (x[row_map[i]] Wu_e^T)
 *                                                               (moe_grouped_swiglu)
 *   down    ys[i] = h[i] Wd_e^T                                 (moe_grouped_down)
 *   combine y[t] = sum_j w[t][j] * ys[inv_order[t*k + j]]       (moe_combine)
 *
 * and all of it in one call (moe_forward).
 *
 * Sources of the operations (the web pages the method is taken from):
 *   - "5.5 real sparse MoE kernels (Metal)" (posttrainllm PRD), section
 *     "Scope -- in": top-K routing kernel (routing_logits -> top_k_indices,
 *     top_k_weights, no host round trip), expert dispatch, post-expert combine.
 *   - mlxcel PR #275, "What it does": out[h] = sum_k scores[k] *
 *     down_k(silu(gate_k(x)) * up_k(x))[h], with affine dequantised experts.
 *   - mlx-lm PR #2044, "What" and "When it applies": experts grouped by expert
 *     so each expert's weights are read and dequantised once per tile; affine
 *     4-bit, group 64; a small-batch regime when tokens per expert T*k/E <= 8.
 *   - DS4Server issue #112, "Current upstream route" and "Kernel contract":
 *     sort_rows (argsort of flattened expert ids, inv_order = argsort(order),
 *     row_map = order // top_k as uint32), swiglu_rows reading token rows in
 *     place through row_map, sorted down projection, _scatter_unsort;
 *     per-expert tile and row prefix tables with the expert found by binary
 *     search; 32-bit row positions.
 *   - MOE_OPTIMIZATION_COMPLETE.md (markbaseengine), "Mega Kernel
 *     Architecture": router matmul, softmax, top-K and dispatch on the GPU
 *     with no CPU wait in between.
 *
 * Conventions shared by every call:
 *   - Pointers marked (device) are CUDA device pointers owned by the caller;
 *     the library never allocates, frees, or keeps them after the call.
 *     Pointers marked (host) are read before the call returns.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream). The library never synchronises the stream and
 *     never reads device data on the host.
 *   - Argument errors are detected on the host before any launch and returned
 *     synchronously; nothing is launched then. MOE_ERR_CUDA reports a launch
 *     error (cudaGetLastError after the launches).
 *   - Device-side errors (a bounded wait that ran out, a value outside the
 *     fp16 range of the expert GEMMs) are recorded in one status word per
 *     device and per process: every call on that device, on any stream or
 *     host thread, reports into the same word, and the first error since
 *     the last read is kept. Read and clear it with moe_device_status().
 *   - T = 0 is valid: the call returns MOE_OK and launches nothing.
 *   - Preconditions: 1 <= k <= min(E, 32); E <= 1024; d and F multiples of 64;
 *     bf16 expert weights need bf16 activations, f32 weights need f32
 *     activations, quantised (q4 / q8) weights take bf16 or fp16 ones. Violations return MOE_ERR_INVALID_ARG or
 *     MOE_ERR_UNSUPPORTED.
 *   - All layouts are row-major with the stated shapes; buffers must be
 *     16-byte aligned.
 *   - Calls are reentrant and keep no state between calls, apart from the
 *     device status word above, the no-allocation sort's scratch array
 *     (moe_sort_rows_noalloc) and the wait bound (moe_set_wait_cycles).
 *   - The library looks up the device addresses of its own device variables
 *     (the status word, the no-allocation scratch) once per device and keeps
 *     them for the life of the process; a cudaDeviceReset() followed by
 *     further calls is not supported.
 *
 * Regimes: moe_grouped_swiglu / moe_grouped_down / moe_forward take a regime.
 *   MOE_REGIME_GEMV: weight-streaming kernels, every selected expert's bytes
 *     read once per step; moe_forward runs the whole layer as one
 *     cooperative launch (the fused decode kernel) where that kernel applies
 *     (q4 experts, T <= 32, T*k <= 256, E <= 256, d and F multiples of 128
 *     up to 2048);
 *   MOE_REGIME_TC: tensor-core grouped GEMM (tcgen05 / TMEM, TMA-staged
 *     operands) for many tokens per expert (prefill); bf16 activations with
 *     bf16 weights, or bf16 / fp16 activations with any quantised format
 *     (q4 groups 32/64/128, q8 group 64); d a multiple of 256, F of 128 (q4:
 *     of 256); other shapes return MOE_ERR_UNSUPPORTED;
 *   MOE_REGIME_AUTO: TC wherever the tensor-core kernels tile the shape
 *     (16-bit activations), except that moe_forward keeps the fused decode
 *     kernel while it applies and T*k < E; GEMV for everything else
 *     (f32 activations, other shapes).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* same type as cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null pointer, negative size, k > E, misaligned ... */
  MOE_ERR_UNSUPPORTED = 2, /* valid but not implemented (dims, dtype/format mix) */
  MOE_ERR_WORKSPACE = 3,   /* workspace pointer null or smaller than required */
  MOE_ERR_CUDA = 4,        /* a CUDA launch failed */
  MOE_ERR_TIMEOUT = 5,     /* a device-side bounded wait ran out (device status) */
  MOE_ERR_RANGE = 6        /* a value outside the fp16 range of the expert GEMMs'
                              operands (|x| or |h| >= 65520; device status) */
} moe_status;

/* activations (x, the router weight, y): fp32, bf16 or IEEE binary16 */
typedef enum { MOE_F32 = 0, MOE_BF16 = 1, MOE_F16 = 2 } moe_dtype;

typedef enum {
  MOE_W_F32 = 0,
  MOE_W_BF16 = 1,
  MOE_W_Q4G64 = 2,
  MOE_W_Q4G32 = 3,   /* as MOE_W_Q4G64 with one scale and bias per 32 elements */
  MOE_W_Q4G128 = 4,  /* ... per 128 elements */
  MOE_W_Q8G64 = 5    /* 8-bit affine, group 64 */
} moe_wfmt;

typedef enum { MOE_REGIME_AUTO = 0, MOE_REGIME_GEMV = 1, MOE_REGIME_TC = 2 } moe_regime;

/* The GLU's gate activation (mlx-lm PR #2044, "When it applies": SwiGLU or
 * tanh-GELU GLU): h = act(gate) * up with
 *   MOE_ACT_SWIGLU:     act(g) = silu(g) = g / (1 + exp(-g))
 *   MOE_ACT_GEGLU_TANH: act(g) = 0.5 g (1 + tanh(sqrt(2/pi) (g + 0.044715 g^3))) */
typedef enum { MOE_ACT_SWIGLU = 0, MOE_ACT_GEGLU_TANH = 1 } moe_act;

/* Expert weights (all device, read-only, caller-owned).
 *   MOE_W_F32 / MOE_W_BF16:
 *     w_gu [E][2F][d]  rows 0..F-1 gate, rows F..2F-1 up (fused [gate|up])
 *     w_dn [E][d][F]
 *     s_* and b_* unused (may be NULL)
 *   MOE_W_Q4G64 (4-bit affine, group 64 along the input dimension;
 *   mlx-lm PR #2044 "When it applies"):
 *     w_gu uint32 [E][2F][d/8], s_gu, b_gu bf16 [E][2F][d/64]
 *     w_dn uint32 [E][d][F/8],  s_dn, b_dn bf16 [E][d][F/64]
 *     element j of a word sits in bits [4j, 4j+3] (low nibble first);
 *     value = scale[group] * q + bias[group].
 *   MOE_W_Q4G32 / MOE_W_Q4G128: the same with groups of 32 or 128 (DS4Server
 *     issue #112, "Kernel contract": group 32/64/128); s_* and b_* are
 *     [E][rows][cols/32] or [E][rows][cols/128]. Every kernel family takes
 *     them (weight-streaming, fused decode, tensor cores).
 *   MOE_W_Q8G64 (8-bit affine; mlxcel PR #275, "Multi-bit handling"; DS4Server
 *   issue #112, "Kernel contract": 4 or 8 bits):
 *     w_gu uint32 [E][2F][d/4], w_dn uint32 [E][d][F/4], byte j of a word is
 *     element j; s_*, b_* bf16 [E][rows][cols/64]; value = scale * q + bias.
 *     It runs on the weight-streaming SIMT kernels and the tensor cores.
 *   Quantised formats: the scale and bias arrays are 16-byte aligned, like
 *     every other buffer.
 *   act: moe_act, the gate activation of every expert (0, SwiGLU, when the
 *     struct is zero-initialised); other values: MOE_ERR_INVALID_ARG. */
typedef struct {
  int32_t fmt; /* moe_wfmt */
  int32_t E, d, F;
  const void* w_gu;
  const void* s_gu;
  const void* b_gu;
  const void* w_dn;
  const void* s_dn;
  const void* b_dn;
  int32_t act; /* moe_act */
} moe_experts;

/* Router: logits, softmax, top-k, renormalised weights.
 * ("5.5 real sparse MoE kernels (Metal)", Scope -- in; "Mega Kernel
 * Architecture" phases 1-3.)
 *   x          (device) [T][d], dtype dt
 *   w_router   (device) [E][d], dtype dt: row e is column e of W_r [d][E]
 *   router_bias(device) [E] fp32, or NULL; added to the logits before the
 *              softmax and the selection
 *   logits     (device, out) [T][E] fp32: x . W_r + b, fp32 accumulation
 *   topk_idx   (device, out) [T][k] int32: selected experts, best first;
 *              ties go to the lowest expert index, -0.0 == +0.0, NaN last
 *   topk_w     (device, out) [T][k] fp32: exp(L_j - max) / sum over selected
 *              (= softmax over all E renormalised over the selection) */
moe_status moe_route(const void* x, moe_dtype dt, const void* w_router, const float* router_bias,
                     int T, int d, int E, int k, float* logits, int32_t* topk_idx, float* topk_w,
                     moe_stream_t stream);

/* Softmax / top-k step alone, from given fp32 logits [T][E] (device).
 * Same outputs and rules as moe_route. */
moe_status moe_topk(const float* logits, int T, int E, int k, int32_t* topk_idx, float* topk_w,
                    moe_stream_t stream);

/* Dispatch: stable counting sort of the R = T*k routed slots r = t*k + j by
 * expert id (DS4Server issue #112, "Current upstream route": sort_rows;
 * "Kernel contract": per-expert tile and row prefix tables).
 *   topk_idx  (device) [T][k] int32, values in [0, E)
 *   BM        rows per tile for tile_off (>= 1)
 *   order     (device, out) [R] uint32: order[i] = slot r of sorted row i;
 *             rows grouped by expert (ascending), slots ascending within one
 *   inv_order (device, out) [R] uint32: inv_order[order[i]] = i
 *   row_map   (device, out) [R] uint32: row_map[i] = order[i] / k (token)
 *   counts    (device, out) [E] int32: rows per expert
 *   row_off   (device, out) [E+1] int32: exclusive scan of counts
 *   tile_off  (device, out) [E+1] int32: exclusive scan of ceil(counts/BM)
 *   ws        (device) scratch of moe_sort_rows_workspace(T, k, E) bytes
 *             (contents on entry do not matter)
 * Ids outside [0, E) are a caller error; the kernels clamp them so that no
 * access leaves the buffers, and the result is then unspecified. */
size_t moe_sort_rows_workspace(int T, int k, int E);
moe_status moe_sort_rows(const int32_t* topk_idx, int T, int k, int E, int BM, uint32_t* order,
                         uint32_t* inv_order, uint32_t* row_map, int32_t* counts, int32_t* row_off,
                         int32_t* tile_off, void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_sort_rows for callers that cannot allocate device memory: the same
 * outputs, bit for bit, with no workspace argument. The source pages have no
 * counterpart to this call. It is meant for code that runs inside a host
 * framework which owns all device memory and hands an operator no allocator
 * or workspace (a plugin or custom-op interface), and for code that must not
 * allocate at the point where it sorts.
 *   Scratch: a static device array inside the library (256 KiB, held by every
 *     GPU that loads the library until the process exits), so sizes are
 *     limited: T*k <= 32768 and E <= 1024, else MOE_ERR_UNSUPPORTED. It calls
 *     no cudaMalloc, cudaFree or any allocating routine.
 *   Set-up: the first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture. MOE_ERR_CUDA if the lookup fails. The
 *     address is kept for the life of the process (see the conventions:
 *     cudaDeviceReset is not supported).
 *   Sharing: every call uses the same array. Calls that may overlap on the
 *     GPU (other streams, other host threads) race and corrupt each other's
 *     result; serialise them. The array keeps the last call's contents; the
 *     sort writes every entry it reads first, so nothing needs clearing.
 * Other arguments and errors: as moe_sort_rows. */
moe_status moe_sort_rows_noalloc(const int32_t* topk_idx, int T, int k, int E, int BM,
                                 uint32_t* order, uint32_t* inv_order, uint32_t* row_map,
                                 int32_t* counts, int32_t* row_off, int32_t* tile_off,
                                 moe_stream_t stream);

/* Grouped gate|up projection with the SwiGLU epilogue over sorted rows,
 * reading token rows in place through row_map (DS4Server issue #112,
 * swiglu_rows; mlxcel PR #275 "What it does").
 *   x        (device) [T][d], dtype dt
 *   row_map, row_off, tile_off: as written by moe_sort_rows with the same BM
 *            (the tensor-core regime needs BM = 128)
 *   h        (device, out) [T*k][F]: fp16 for 16-bit activations, fp32 for fp32:
 *            h[i][f] = act(g) * u (experts->act: silu or tanh-GELU),
 *            g = x[row_map[i]] . w_gu[e][f],
 *            u = x[row_map[i]] . w_gu[e][F+f], e = expert of row i
 *   ws       (device) scratch of moe_grouped_swiglu_workspace(T, k, d, dt)
 *            bytes (the token rows in 16 bits: x converted to fp16, or, in
 *            the tensor-core regime, gathered into sorted row order); required
 *            for 16-bit activations, may be NULL for fp32
 * fp32 accumulation; h rounded once. The tensor-core regime multiplies fp16
 * operands (fp16 x as is, bf16 x converted exactly when |x| < 65520, weights
 * dequantised to fp16); values outside fp16 range are reported as
 * MOE_ERR_RANGE in the device status. bf16 experts with bf16 activations are
 * multiplied as bf16 (the same products, exact in fp32; no range limit on
 * x). */
size_t moe_grouped_swiglu_workspace(int T, int k, int d, moe_dtype dt);
moe_status moe_grouped_swiglu(const void* x, moe_dtype dt, const uint32_t* row_map,
                              const int32_t* row_off, const int32_t* tile_off, int BM, int T, int k,
                              const moe_experts* experts, void* h, void* ws, size_t ws_bytes,
                              moe_regime regime, moe_stream_t stream);

/* Grouped down projection over rows already sorted by expert (DS4Server
 * issue #112, switch_linear with sorted indices).
 *   h        (device) [T*k][F]: fp16 for 16-bit activations (MOE_BF16, MOE_F16),
 *            fp32 for fp32 -- as moe_grouped_swiglu writes it
 *   ys       (device, out) [T*k][d]: ys[i][o] = h[i] . w_dn[e][o], fp32
 *            accumulation, stored in fp16 for 16-bit activations (its 11-bit
 *            rounding is far below the final bf16 rounding of y; values
 *            outside fp16 range are reported as MOE_ERR_RANGE in the device
 *            status) and in fp32 for fp32 activations */
moe_status moe_grouped_down(const void* h, moe_dtype dt, const int32_t* row_off,
                            const int32_t* tile_off, int BM, int T, int k,
                            const moe_experts* experts, void* ys, moe_regime regime,
                            moe_stream_t stream);

/* Score-weighted unsort back to token order, atomic-free (DS4Server issue
 * #112, _scatter_unsort; "5.5 real sparse MoE kernels (Metal)", scatter_add
 * equivalent): y[t][o] = sum_{j=0..k-1} w[t][j] * ys[inv_order[t*k+j]][o],
 * summed in fp32 in j order, rounded once to dt.
 *   ys (device) [T*k][d]: fp16 for MOE_BF16 / MOE_F16, fp32 for MOE_F32 (as
 *      moe_grouped_down writes it); inv_order (device) [T*k];
 *      topk_w (device) [T][k] fp32
 *   y  (device, out) [T][d], dtype dt */
moe_status moe_combine(const void* ys, const uint32_t* inv_order, const float* topk_w, int T, int k,
                       int d, moe_dtype dt, void* y, moe_stream_t stream);

/* The whole layer in one call, on one stream, no host synchronisation
 * (MOE_OPTIMIZATION_COMPLETE.md, "Mega Kernel Architecture": no CPU wait
 * between router and experts).
 *   x, w_router, router_bias: as for moe_route; experts: as above
 *   y   (device, out) [T][d], dtype dt
 *   ws  (device) workspace of moe_forward_workspace(...) bytes; it holds the
 *       intermediates at the offsets moe_forward_layout() reports */
size_t moe_forward_workspace(int T, int d, int E, int k, int F, moe_dtype dt, moe_wfmt wfmt,
                             moe_regime regime);
moe_status moe_forward(const void* x, moe_dtype dt, const void* w_router, const float* router_bias,
                       const moe_experts* experts, int T, int k, void* y, void* ws,
                       size_t ws_bytes, moe_regime regime, moe_stream_t stream);

/* Where moe_forward keeps each intermediate inside its workspace (byte
 * offsets), the regime it resolves to for experts of weight format wfmt and
 * the BM it sorts with. moe_forward_workspace(...) is its `total`; 0 when the
 * arguments are invalid. x16 holds 16-bit token rows: fp16, or bf16 as
 * given for bf16 experts with bf16 activations on the tensor cores. With q4
 * experts the whole-layer call may keep h and x16 with every 8 consecutive
 * elements in the order (0, 4, 1, 5, 2, 6, 3, 7), the K order its kernels
 * dequantise in; the routing and sort tables have the layouts moe_route and
 * moe_sort_rows give. */
typedef struct {
  size_t logits, topk_idx, topk_w, order, inv_order, row_map, counts, row_off, tile_off;
  size_t sort_ws, h, ys, x16, total;
  int32_t regime; /* resolved: MOE_REGIME_GEMV or MOE_REGIME_TC */
  int32_t BM;
} moe_ws_layout;
moe_status moe_forward_layout(int T, int d, int E, int k, int F, moe_dtype dt, moe_wfmt wfmt,
                              moe_regime regime, moe_ws_layout* out /* (host, out) */);

/* Token rows per tile (BM) of the tensor-core regime: moe_grouped_swiglu and
 * moe_grouped_down in that regime need tile_off written by moe_sort_rows with
 * this BM (DS4Server issue #112, "Kernel contract": per-expert tile prefix
 * table). The weight-streaming regime takes any BM >= 1. */
int moe_sort_block_m(void);

/* Read the current device's status word (MOE_OK or the first device-side
 * error since the last read, from any stream) and reset it. Synchronises the
 * current device. */
moe_status moe_device_status(void);

/* Bound of the device-side waits, in SM cycles. Every kernel that waits
 * (for a copy, an MMA, another warp role or another CTA) gives up after this
 * many cycles, records MOE_ERR_TIMEOUT in the device status word, finishes
 * the copies and MMAs it has in flight, releases its tensor memory and
 * returns; the caller reads the status with moe_device_status(). The bound is
 * one value for the whole process, read by every launch after the call. 0
 * restores the default, 2e9 cycles (about one second at the B200's clocks);
 * a short bound is for tests that make the waits of a real forward run out.
 * The source pages have no counterpart to this call.
 * Negative values: MOE_ERR_INVALID_ARG. */
moe_status moe_set_wait_cycles(long long cycles);

/* Test support, no counterpart on the source pages: launches a one-block
 * kernel whose single wait can never be satisfied, with a bound of `cycles`
 * (>= 1), using the library's own wait code, so that a test can see a
 * bounded wait run out and the kernel return with MOE_ERR_TIMEOUT recorded
 * in the device status word.
 *   which 0: the mbarrier wait of the tensor-core grouped kernels;
 *         1: the mbarrier wait of the fused decode kernel;
 *         2: the grid barrier of the fused decode kernel; scratch (device,
 *            16-byte aligned, >= 4 bytes) holds its counter
 * Asynchronous on `stream`; MOE_OK when launched. */
moe_status moe_selftest_wait_timeout(int which, long long cycles, void* scratch,
                                     moe_stream_t stream);

/* Pack separate gate and up projections into the fused [gate|up] layout the
 * kernels read (w_gu rows 0..F-1 gate, F..2F-1 up of every expert).
 * DS4Server issue #112, "Kernel contract", takes both the fused [gate | up]
 * weight and separate gate/up weights; here separate weights are packed once,
 * at load time, rather than streamed as two tensors in every kernel.
 *   fmt            moe_wfmt of all six tensors
 *   w_g, w_u       (device) [E][F][d] (f32/bf16) or uint32 [E][F][d/8] (q4)
 *   s_g, b_g, s_u, b_u (device) q4 only: bf16 [E][F][d/64]; else ignored
 *   w_gu, s_gu, b_gu   (device, out) the fused tensors, [E][2F][...]
 * One strided device-to-device copy per tensor on `stream`; nothing is
 * allocated. d and F are multiples of 64; E, d, F > 0; the outputs must not
 * overlap the inputs. */
moe_status moe_pack_gate_up(int fmt, int E, int d, int F, const void* w_g, const void* s_g,
                            const void* b_g, const void* w_u, const void* s_u, const void* b_u,
                            void* w_gu, void* s_gu, void* b_gu, moe_stream_t stream);

const char* moe_status_str(moe_status s);
const char* moe_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
