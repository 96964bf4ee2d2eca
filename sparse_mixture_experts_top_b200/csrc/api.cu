// C ABI entry points: argument checks, workspace carving, launch sequences.
// Every check runs on the host before the first launch; nothing here reads
// device memory or synchronises a stream (except moe_device_status).
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace moe {

__device__ int g_moe_status;   // first device-side error since the last read

static int* status_ptr() {
  static std::mutex mu;
  static int* ptrs[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_moe_status) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<int*>(p);
  }
  return ptrs[dev];
}

// bound of every device-side wait for work, in SM cycles; 0 = the default
static std::atomic<long long> g_wait_cycles{0};

long long wait_cycles() {
  const long long v = g_wait_cycles.load(std::memory_order_relaxed);
  return v > 0 ? v : kDefaultWaitCycles;
}

static inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static inline size_t up256(size_t v) { return (v + 255) & ~(size_t)255; }
static inline size_t act_size(int dt) { return dt == MOE_F32 ? 4 : 2; }

static moe_status launched(cudaError_t e) {
  if (e == cudaSuccess) return MOE_OK;
  if (e == cudaErrorInvalidValue || e == cudaErrorNotSupported) return MOE_ERR_UNSUPPORTED;
  return MOE_ERR_CUDA;
}

static moe_status check_dims(int T, int d, int E, int k) {
  if (T < 0 || d <= 0 || E <= 0 || k <= 0 || k > E) return MOE_ERR_INVALID_ARG;
  if (k > 32 || E > 1024) return MOE_ERR_UNSUPPORTED;
  if ((long long)T * k > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

static moe_status check_experts(const moe_experts* ex, int dt) {
  if (!ex) return MOE_ERR_INVALID_ARG;
  if (ex->E <= 0 || ex->d <= 0 || ex->F <= 0) return MOE_ERR_INVALID_ARG;
  if (ex->d % 64 || ex->F % 64) return MOE_ERR_UNSUPPORTED;
  if (!ex->w_gu || !ex->w_dn) return MOE_ERR_INVALID_ARG;
  if (!aligned16(ex->w_gu) || !aligned16(ex->w_dn)) return MOE_ERR_INVALID_ARG;
  if (ex->act != MOE_ACT_SWIGLU && ex->act != MOE_ACT_GEGLU_TANH) return MOE_ERR_INVALID_ARG;
  switch (ex->fmt) {
    case MOE_W_F32:
      if (dt != MOE_F32) return MOE_ERR_UNSUPPORTED;
      break;
    case MOE_W_BF16:
      if (dt != MOE_BF16) return MOE_ERR_UNSUPPORTED;
      break;
    case MOE_W_Q4G64:
    case MOE_W_Q4G32:
    case MOE_W_Q4G128:
      if (dt == MOE_F32) return MOE_ERR_UNSUPPORTED;
      if (!ex->s_gu || !ex->b_gu || !ex->s_dn || !ex->b_dn) return MOE_ERR_INVALID_ARG;
      if (!aligned16(ex->s_gu) || !aligned16(ex->b_gu) || !aligned16(ex->s_dn) ||
          !aligned16(ex->b_dn))
        return MOE_ERR_INVALID_ARG;
      if (ex->d % q4_group(ex->fmt) || ex->F % q4_group(ex->fmt)) return MOE_ERR_UNSUPPORTED;
      break;
    case MOE_W_Q8G64:
      if (dt == MOE_F32) return MOE_ERR_UNSUPPORTED;
      if (!ex->s_gu || !ex->b_gu || !ex->s_dn || !ex->b_dn) return MOE_ERR_INVALID_ARG;
      if (!aligned16(ex->s_gu) || !aligned16(ex->b_gu) || !aligned16(ex->s_dn) ||
          !aligned16(ex->b_dn))
        return MOE_ERR_INVALID_ARG;
      break;
    default:
      return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

static bool valid_dt(int dt) { return dt == MOE_F32 || dt == MOE_BF16 || dt == MOE_F16; }

// The regime a call runs. AUTO takes the tensor-core kernels wherever they
// tile the shape (16-bit activations; d % 256, F % 128, or % 256 for q4;
// q4, q8 or bf16 weights), except that the whole-layer call keeps the
// one-launch fused decode kernel while it applies and fewer than E rows are
// routed; the weight-streaming kernels take everything else. Measured on one
// B200 (graph-replayed forwards, L2 flushed): at E = 128, top-8, F = 768 the
// fused kernel is faster up to 12 tokens (84 against 92 us at 8, 110 against
// 116 at 12) and the tensor cores from 16 (117 against 124 us; 138 against
// 166 at 32); at E = 512, top-10, where the fused kernel does not apply, the
// tensor cores are faster from 4 tokens (60 against 76 us); with 8 bf16
// experts from 1 token (86 against 107 us).
static int resolve_regime(int regime, long long R, int E, int dt, int d, int F, int fmt,
                          bool fused_decode) {
  if (regime == MOE_REGIME_GEMV || regime == MOE_REGIME_TC) return regime;
  if (dt == MOE_F32 || !tc_shape_supported(d, F, fmt, dt)) return MOE_REGIME_GEMV;
  if (fused_decode && R < E) return MOE_REGIME_GEMV;
  return MOE_REGIME_TC;
}

static int block_m_for(int regime, long long R, int E) {
  if (regime == MOE_REGIME_TC) return tc_block_m();
  return (R <= 8LL * E) ? 16 : 32;
}

// gate|up in the weight-streaming regime: the q4 tensor-core GEMV when it
// applies (bf16 x converted to fp16 into x16 first; fp16 x read in place),
// else the SIMT kernel
static cudaError_t swiglu_gemv(const void* x, int dt, int T, const uint32_t* rmap,
                               const int32_t* roff, const int32_t* toff, int BM, int R,
                               const moe_experts& ex, void* h, void* x16, int* stp,
                               cudaStream_t s) {
  if (gemv_q4_mma_ok(ex, dt, BM) && dt == MOE_F16)
    return launch_swiglu_q4_mma(x, rmap, roff, toff, BM, R, ex, h, stp, s);
  if (gemv_q4_mma_ok(ex, dt, BM) && x16) {
    cudaError_t e = launch_to_f16(x, (long long)T * ex.d, x16, stp, s);
    if (e != cudaSuccess) return e;
    return launch_swiglu_q4_mma(x16, rmap, roff, toff, BM, R, ex, h, stp, s);
  }
  return launch_swiglu_gemv(x, dt, rmap, roff, toff, BM, R, ex, h, stp, s);
}

static cudaError_t down_gemv(const void* h, int dt, const int32_t* roff, const int32_t* toff,
                             int BM, int R, const moe_experts& ex, void* ys, int* stp,
                             cudaStream_t s) {
  if (gemv_q4_mma_ok(ex, dt, BM)) return launch_down_q4_mma(h, roff, toff, BM, R, ex, ys, stp, s);
  return launch_down_gemv(h, dt, roff, toff, BM, R, ex, ys, stp, s);
}

}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_version(void) { return "moe-b200 0.1 (sm_100a)"; }

const char* moe_status_str(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape, dtype or format";
    case MOE_ERR_WORKSPACE: return "workspace missing or too small";
    case MOE_ERR_CUDA: return "CUDA launch error";
    case MOE_ERR_TIMEOUT: return "device-side bounded wait ran out";
    case MOE_ERR_RANGE: return "value outside the fp16 range of the expert GEMM operands";
  }
  return "unknown status";
}

moe_status moe_device_status(void) {
  int* p = status_ptr();
  if (!p) return MOE_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return MOE_ERR_CUDA;
  return (moe_status)v;
}

moe_status moe_set_wait_cycles(long long cycles) {
  if (cycles < 0) return MOE_ERR_INVALID_ARG;
  g_wait_cycles.store(cycles, std::memory_order_relaxed);
  return MOE_OK;
}

moe_status moe_selftest_wait_timeout(int which, long long cycles, void* scratch,
                                     moe_stream_t stream) {
  if (which < 0 || which > 2 || cycles < 1) return MOE_ERR_INVALID_ARG;
  if (which == 2 && (!scratch || !aligned16(scratch))) return MOE_ERR_INVALID_ARG;
  int* stp = status_ptr();
  if (!stp) return MOE_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  if (which == 0) return launched(launch_tc_wait_selftest(cycles, stp, s));
  return launched(launch_decode_wait_selftest(which, cycles, (unsigned*)scratch, stp, s));
}

moe_status moe_topk(const float* logits, int T, int E, int k, int32_t* topk_idx, float* topk_w,
                    moe_stream_t stream) {
  moe_status st = check_dims(T, 64, E, k);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!logits || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  return launched(launch_topk(logits, T, E, k, topk_idx, topk_w, (cudaStream_t)stream));
}

moe_status moe_route(const void* x, moe_dtype dt, const void* w_router, const float* router_bias,
                     int T, int d, int E, int k, float* logits, int32_t* topk_idx, float* topk_w,
                     moe_stream_t stream) {
  moe_status st = check_dims(T, d, E, k);
  if (st != MOE_OK) return st;
  if (!valid_dt(dt)) return MOE_ERR_INVALID_ARG;
  if (d % 64) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!x || !w_router || !logits || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_router)) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaErrorNotSupported;
  if (dt != MOE_F32) e = launch_router_logits_tc(x, dt, w_router, router_bias, T, d, E, logits,
                                                 status_ptr(), s);
  if (e == cudaErrorNotSupported)
    e = launch_router_logits(x, dt, w_router, router_bias, T, d, E, logits, s);
  if (e != cudaSuccess) return launched(e);
  return launched(launch_topk(logits, T, E, k, topk_idx, topk_w, s));
}

size_t moe_sort_rows_workspace(int T, int k, int E) {
  if (T < 0 || k <= 0 || E <= 0) return 0;
  return sort_workspace_bytes((int)((long long)T * k), E);
}

moe_status moe_sort_rows(const int32_t* topk_idx, int T, int k, int E, int BM, uint32_t* order,
                         uint32_t* inv_order, uint32_t* row_map, int32_t* counts, int32_t* row_off,
                         int32_t* tile_off, void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_dims(T, 64, E, k);
  if (st != MOE_OK) return st;
  if (BM < 1) return MOE_ERR_INVALID_ARG;
  if (!counts || !row_off || !tile_off) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!topk_idx || !order || !inv_order || !row_map)) return MOE_ERR_INVALID_ARG;
  const long long R = (long long)T * k;
  if (R > 1024) {
    if (!ws) return MOE_ERR_WORKSPACE;
    if (ws_bytes < moe_sort_rows_workspace(T, k, E)) return MOE_ERR_WORKSPACE;
  }
  return launched(launch_sort_rows(topk_idx, T, k, E, BM, order, inv_order, row_map, counts,
                                   row_off, tile_off, ws, (cudaStream_t)stream));
}

size_t moe_grouped_swiglu_workspace(int T, int k, int d, moe_dtype dt) {
  if (T < 0 || k < 1 || d <= 0) return 0;
  // fp16 token rows: T rows (weight-streaming regime) or the T*k rows in
  // sorted order (tensor-core regime)
  return dt != MOE_F32 ? up256((size_t)T * k * d * 2) : 0;
}

moe_status moe_sort_rows_noalloc(const int32_t* topk_idx, int T, int k, int E, int BM,
                                 uint32_t* order, uint32_t* inv_order, uint32_t* row_map,
                                 int32_t* counts, int32_t* row_off, int32_t* tile_off,
                                 moe_stream_t stream) {
  moe_status st = check_dims(T, 64, E, k);
  if (st != MOE_OK) return st;
  if (BM < 1) return MOE_ERR_INVALID_ARG;
  if (!counts || !row_off || !tile_off) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!topk_idx || !order || !inv_order || !row_map)) return MOE_ERR_INVALID_ARG;
  if (!noalloc_sort_fits((long long)T * k, E)) return MOE_ERR_UNSUPPORTED;
  return launched(launch_sort_rows_noalloc(topk_idx, T, k, E, BM, order, inv_order, row_map,
                                           counts, row_off, tile_off, (cudaStream_t)stream));
}

moe_status moe_grouped_swiglu(const void* x, moe_dtype dt, const uint32_t* row_map,
                              const int32_t* row_off, const int32_t* tile_off, int BM, int T, int k,
                              const moe_experts* experts, void* h, void* ws, size_t ws_bytes,
                              moe_regime regime, moe_stream_t stream) {
  if (!valid_dt(dt)) return MOE_ERR_INVALID_ARG;
  moe_status st = check_experts(experts, dt);
  if (st != MOE_OK) return st;
  st = check_dims(T, experts->d, experts->E, k);
  if (st != MOE_OK) return st;
  if (BM < 1) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !row_map || !row_off || !tile_off || !h) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(h)) return MOE_ERR_INVALID_ARG;
  const long long R = (long long)T * k;
  const int rg = resolve_regime(regime, R, experts->E, dt, experts->d, experts->F, experts->fmt,
                                false);
  cudaStream_t s = (cudaStream_t)stream;
  if (rg == MOE_REGIME_TC) {
    if (dt == MOE_F32) return MOE_ERR_UNSUPPORTED;
    if (!tc_shape_supported(experts->d, experts->F, experts->fmt, dt)) return MOE_ERR_UNSUPPORTED;
    if (BM != tc_block_m()) return MOE_ERR_INVALID_ARG;
    if (!ws || !aligned16(ws) || ws_bytes < moe_grouped_swiglu_workspace(T, k, experts->d, dt))
      return MOE_ERR_WORKSPACE;
    return launched(launch_swiglu_tc(x, dt, T, row_map, row_off, tile_off, (int)R, *experts, h, ws,
                                     status_ptr(), s));
  }
  if (dt != MOE_F32 &&
      (!ws || !aligned16(ws) || ws_bytes < moe_grouped_swiglu_workspace(T, k, experts->d, dt)))
    return MOE_ERR_WORKSPACE;
  return launched(swiglu_gemv(x, dt, T, row_map, row_off, tile_off, BM, (int)R, *experts, h, ws,
                              status_ptr(), s));
}

moe_status moe_grouped_down(const void* h, moe_dtype dt, const int32_t* row_off,
                            const int32_t* tile_off, int BM, int T, int k,
                            const moe_experts* experts, void* ys, moe_regime regime,
                            moe_stream_t stream) {
  if (!valid_dt(dt)) return MOE_ERR_INVALID_ARG;
  moe_status st = check_experts(experts, dt);
  if (st != MOE_OK) return st;
  st = check_dims(T, experts->d, experts->E, k);
  if (st != MOE_OK) return st;
  if (BM < 1) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!h || !row_off || !tile_off || !ys) return MOE_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(ys)) return MOE_ERR_INVALID_ARG;
  const long long R = (long long)T * k;
  const int rg = resolve_regime(regime, R, experts->E, dt, experts->d, experts->F, experts->fmt,
                                false);
  cudaStream_t s = (cudaStream_t)stream;
  if (rg == MOE_REGIME_TC) {
    if (dt == MOE_F32) return MOE_ERR_UNSUPPORTED;
    if (!tc_shape_supported(experts->d, experts->F, experts->fmt, dt)) return MOE_ERR_UNSUPPORTED;
    if (BM != tc_block_m()) return MOE_ERR_INVALID_ARG;
    return launched(launch_down_tc(h, row_off, tile_off, (int)R, *experts, ys, status_ptr(), s));
  }
  return launched(down_gemv(h, dt, row_off, tile_off, BM, (int)R, *experts, ys, status_ptr(), s));
}

moe_status moe_combine(const void* ys, const uint32_t* inv_order, const float* topk_w, int T, int k,
                       int d, moe_dtype dt, void* y, moe_stream_t stream) {
  if (!valid_dt(dt)) return MOE_ERR_INVALID_ARG;
  if (T < 0 || k <= 0 || d <= 0) return MOE_ERR_INVALID_ARG;
  if (k > 32) return MOE_ERR_UNSUPPORTED;
  if (d % 64) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!ys || !inv_order || !topk_w || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned16(ys) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  return launched(launch_combine(ys, inv_order, topk_w, T, k, d, dt, y, (cudaStream_t)stream));
}

moe_status moe_pack_gate_up(int fmt, int E, int d, int F, const void* w_g, const void* s_g,
                            const void* b_g, const void* w_u, const void* s_u, const void* b_u,
                            void* w_gu, void* s_gu, void* b_gu, moe_stream_t stream) {
  if (E <= 0 || d <= 0 || F <= 0) return MOE_ERR_INVALID_ARG;
  if (d % 64 || F % 64) return MOE_ERR_UNSUPPORTED;
  if (!w_g || !w_u || !w_gu) return MOE_ERR_INVALID_ARG;
  size_t row_bytes = 0;          // bytes of one weight row of d inputs
  switch (fmt) {
    case MOE_W_F32: row_bytes = (size_t)d * 4; break;
    case MOE_W_BF16: row_bytes = (size_t)d * 2; break;
    case MOE_W_Q4G64:
    case MOE_W_Q4G32:
    case MOE_W_Q4G128:
    case MOE_W_Q8G64:
      row_bytes = fmt == MOE_W_Q8G64 ? (size_t)d : (size_t)d / 2;
      if (d % wq_group(fmt)) return MOE_ERR_UNSUPPORTED;
      if (!s_g || !b_g || !s_u || !b_u || !s_gu || !b_gu) return MOE_ERR_INVALID_ARG;
      break;
    default: return MOE_ERR_INVALID_ARG;
  }
  cudaStream_t s = (cudaStream_t)stream;
  // expert e's F gate rows go to rows 0..F-1 of its 2F-row block, its F up
  // rows to rows F..2F-1: a 2-D copy of E blocks of F rows each
  auto pack = [&](const void* g, const void* u, void* out, size_t rb) -> cudaError_t {
    const size_t blk = (size_t)F * rb;
    cudaError_t e = cudaMemcpy2DAsync(out, 2 * blk, g, blk, blk, (size_t)E,
                                      cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return e;
    return cudaMemcpy2DAsync(static_cast<char*>(out) + blk, 2 * blk, u, blk, blk, (size_t)E,
                             cudaMemcpyDeviceToDevice, s);
  };
  cudaError_t e = pack(w_g, w_u, w_gu, row_bytes);
  if (e == cudaSuccess && wq_group(fmt)) {
    const size_t srb = (size_t)(d / wq_group(fmt)) * 2;   // one row's bf16 scales (or biases)
    e = pack(s_g, s_u, s_gu, srb);
    if (e == cudaSuccess) e = pack(b_g, b_u, b_gu, srb);
  }
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_sort_block_m(void) { return tc_block_m(); }

moe_status moe_forward_layout(int T, int d, int E, int k, int F, moe_dtype dt, moe_wfmt wfmt,
                              moe_regime regime, moe_ws_layout* out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  if (!valid_dt(dt)) return MOE_ERR_INVALID_ARG;
  if (wfmt < MOE_W_F32 || wfmt > MOE_W_Q8G64) return MOE_ERR_INVALID_ARG;
  moe_status st = check_dims(T, d, E, k);
  if (st != MOE_OK) return st;
  if (F <= 0) return MOE_ERR_INVALID_ARG;
  if (regime != MOE_REGIME_AUTO && regime != MOE_REGIME_GEMV && regime != MOE_REGIME_TC)
    return MOE_ERR_INVALID_ARG;
  const long long R = (long long)T * k;
  const size_t a = act_size(dt);
  moe_ws_layout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = up256(off + bytes);
    return at;
  };
  L.logits = take((size_t)T * E * 4);
  L.topk_idx = take((size_t)R * 4);
  L.topk_w = take((size_t)R * 4);
  L.order = take((size_t)R * 4);
  L.inv_order = take((size_t)R * 4);
  L.row_map = take((size_t)R * 4);
  L.counts = take((size_t)E * 4);
  L.row_off = take((size_t)(E + 1) * 4);
  L.tile_off = take((size_t)(E + 1) * 4);
  L.sort_ws = take(sort_workspace_bytes((int)R, E));
  L.h = take((size_t)R * F * a);      // fp16 (16-bit activations) or fp32
  L.ys = take((size_t)R * d * a);     // fp16 (16-bit activations) or fp32
  L.regime = resolve_regime(regime, R, E, dt, d, F, wfmt, decode_fused_ok(T, k, E, d, F, wfmt, dt));
  L.BM = block_m_for(L.regime, R, E);
  // fp16 token rows: x converted (weight-streaming), or permuted (the
  // one-launch path), or gathered in sorted row order (tensor cores)
  L.x16 = take(dt == MOE_F32 ? 0 : (size_t)(L.regime == MOE_REGIME_TC ? R : T) * d * 2);
  L.total = off;
  *out = L;
  return MOE_OK;
}

size_t moe_forward_workspace(int T, int d, int E, int k, int F, moe_dtype dt, moe_wfmt wfmt,
                             moe_regime regime) {
  moe_ws_layout L;
  if (moe_forward_layout(T, d, E, k, F, dt, wfmt, regime, &L) != MOE_OK) return 0;
  return L.total;
}

moe_status moe_forward(const void* x, moe_dtype dt, const void* w_router, const float* router_bias,
                       const moe_experts* experts, int T, int k, void* y, void* ws,
                       size_t ws_bytes, moe_regime regime, moe_stream_t stream) {
  if (!valid_dt(dt)) return MOE_ERR_INVALID_ARG;
  moe_status st = check_experts(experts, dt);
  if (st != MOE_OK) return st;
  const int d = experts->d, E = experts->E, F = experts->F;
  st = check_dims(T, d, E, k);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!x || !w_router || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  moe_ws_layout L;
  st = moe_forward_layout(T, d, E, k, F, dt, (moe_wfmt)experts->fmt, regime, &L);
  if (st != MOE_OK) return st;
  if (!ws || !aligned16(ws)) return MOE_ERR_WORKSPACE;
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  // AUTO resolves to TC only for shapes and formats the tensor-core kernels
  // tile; an explicit TC request for others is refused
  const int regime_run = L.regime;
  if (regime_run == MOE_REGIME_TC && !tc_shape_supported(d, F, experts->fmt, dt))
    return MOE_ERR_UNSUPPORTED;

  char* base = static_cast<char*>(ws);
  float* logits = (float*)(base + L.logits);
  int32_t* idx = (int32_t*)(base + L.topk_idx);
  float* w = (float*)(base + L.topk_w);
  uint32_t* order = (uint32_t*)(base + L.order);
  uint32_t* inv = (uint32_t*)(base + L.inv_order);
  uint32_t* rmap = (uint32_t*)(base + L.row_map);
  int32_t* counts = (int32_t*)(base + L.counts);
  int32_t* roff = (int32_t*)(base + L.row_off);
  int32_t* toff = (int32_t*)(base + L.tile_off);
  void* sws = base + L.sort_ws;
  void* h = base + L.h;
  void* ys = base + L.ys;
  void* x16 = base + L.x16;
  const long long R = (long long)T * k;
  cudaStream_t s = (cudaStream_t)stream;
  int* stp = status_ptr();

  cudaError_t e = cudaErrorNotSupported;
  // few tokens: the whole layer in one cooperative launch (its grid barrier
  // counter lives in the sort scratch, which that path does not use)
  if (regime_run == MOE_REGIME_GEMV && decode_fused_ok(T, k, E, d, F, experts->fmt, dt)) {
    e = launch_decode_fused(x, dt, w_router, router_bias, *experts, T, k, L.BM, logits, idx, w, order,
                            inv, rmap, counts, roff, toff, x16, h, ys, y, (unsigned*)sws, stp, s);
    if (e != cudaErrorNotSupported) return launched(e);
  }
  if (dt != MOE_F32) e = launch_router_logits_tc(x, dt, w_router, router_bias, T, d, E, logits, stp, s);
  if (e == cudaErrorNotSupported)
    e = launch_router_logits(x, dt, w_router, router_bias, T, d, E, logits, s);
  if (e != cudaSuccess) return launched(e);
  if ((e = launch_topk(logits, T, E, k, idx, w, s)) != cudaSuccess) return launched(e);
  if ((e = launch_sort_rows(idx, T, k, E, L.BM, order, inv, rmap, counts, roff, toff, sws, s)) !=
      cudaSuccess)
    return launched(e);
  if (regime_run == MOE_REGIME_TC) {
    // h stays in the q4 dequant's permuted K order between the two kernels
    if ((e = launch_swiglu_tc(x, dt, T, rmap, roff, toff, (int)R, *experts, h, x16, stp, s,
                              true)) != cudaSuccess)
      return launched(e);
    if ((e = launch_down_tc(h, roff, toff, (int)R, *experts, ys, stp, s, true)) != cudaSuccess)
      return launched(e);
  } else {
    if ((e = swiglu_gemv(x, dt, T, rmap, roff, toff, L.BM, (int)R, *experts, h,
                         dt == MOE_F32 ? nullptr : x16, stp, s)) != cudaSuccess)
      return launched(e);
    if ((e = down_gemv(h, dt, roff, toff, L.BM, (int)R, *experts, ys, stp, s)) != cudaSuccess)
      return launched(e);
  }
  return launched(launch_combine(ys, inv, w, T, k, d, dt, y, s));
}

}  // extern "C"
