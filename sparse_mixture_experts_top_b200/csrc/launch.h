// Host-side launchers of the MoE forward kernels (internal to the library).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// SM cycles a device-side wait for work may take before the kernel records
// MOE_ERR_TIMEOUT and aborts (moe_set_wait_cycles; about one second unless set)
constexpr long long kDefaultWaitCycles = 2000000000LL;
long long wait_cycles();

// Test support: make one kind of bounded wait run out (see moe_selftest_wait_timeout)
cudaError_t launch_tc_wait_selftest(long long limit, int* status, cudaStream_t s);
cudaError_t launch_decode_wait_selftest(int which, long long limit, unsigned* ctr, int* status,
                                        cudaStream_t s);

// Router logits L[T][E] = x[T][d] . w_router[E][d]^T + bias, fp32 out.
cudaError_t launch_router_logits(const void* x, int dt, const void* w_router, const float* bias,
                                 int T, int d, int E, float* logits, cudaStream_t s);
// Tensor-core router (bf16 or fp16 x and router weight); returns
// cudaErrorNotSupported when the shape is outside what the kernel tiles
// (caller then uses the SIMT one).
cudaError_t launch_router_logits_tc(const void* x, int dt, const void* w_router, const float* bias, int T,
                                    int d, int E, float* logits, int* status, cudaStream_t s);

cudaError_t launch_topk(const float* logits, int T, int E, int k, int32_t* idx, float* w,
                        cudaStream_t s);

size_t sort_workspace_bytes(int R, int E);
cudaError_t launch_sort_rows(const int32_t* idx, int T, int k, int E, int BM, uint32_t* order,
                             uint32_t* inv_order, uint32_t* row_map, int32_t* counts,
                             int32_t* row_off, int32_t* tile_off, void* ws, cudaStream_t s);

// The same sort with its scratch in a static device array (no allocation).
bool noalloc_sort_fits(long long R, int E);
cudaError_t launch_sort_rows_noalloc(const int32_t* idx, int T, int k, int E, int BM,
                                     uint32_t* order, uint32_t* inv_order, uint32_t* row_map,
                                     int32_t* counts, int32_t* row_off, int32_t* tile_off,
                                     cudaStream_t s);

// Upper bound of tile_off[E] for R rows, E experts and BM rows per tile.
inline long long max_tiles(long long R, int E, int BM) {
  long long a = (R + BM - 1) / BM + (R < E ? R : E);
  return a < R ? a : R;
}

// Weight-streaming grouped kernels (any format, any BM).
cudaError_t launch_swiglu_gemv(const void* x, int dt, const uint32_t* row_map,
                               const int32_t* row_off, const int32_t* tile_off, int BM, int R,
                               const moe_experts& ex, void* h, int* status, cudaStream_t s);
cudaError_t launch_down_gemv(const void* h, int dt, const int32_t* row_off,
                             const int32_t* tile_off, int BM, int R, const moe_experts& ex,
                             void* ys, int* status, cudaStream_t s);

// q4 weights with 16-bit activations and at most 16 rows per tile: mma.sync
// fp16 GEMV (x16: fp16 activations, converted from bf16 or the caller's own;
// h fp16 in, ys fp16 out).
bool gemv_q4_mma_ok(const moe_experts& ex, int dt, int BM);
cudaError_t launch_swiglu_q4_mma(const void* x16, const uint32_t* row_map, const int32_t* row_off,
                                 const int32_t* tile_off, int BM, int R, const moe_experts& ex,
                                 void* h, int* status, cudaStream_t s);
cudaError_t launch_down_q4_mma(const void* h, const int32_t* row_off, const int32_t* tile_off,
                               int BM, int R, const moe_experts& ex, void* ys, int* status,
                               cudaStream_t s);
// bf16 -> fp16 copy of n values (n a multiple of 8); out-of-range values
// are reported as MOE_ERR_RANGE
cudaError_t launch_to_f16(const void* x, long long n, void* x16, int* status, cudaStream_t s);

// Tensor-core grouped kernels (bf16 activations with bf16 or q4 weights,
// fp16 activations with q4 weights). BM must equal tc_block_m().
int tc_block_m();
// whether the tensor-core kernels tile these expert shapes and types
bool tc_shape_supported(int d, int F, int fmt, int dt);
// xs16: R*d fp16 scratch that receives the token rows of the R sorted rows,
// gathered through row_map (converted when x is bf16)
// h_perm (q4 experts): h kept in the permuted K order of the q4 dequant
// between the two calls (the whole-layer call); otherwise feature order
cudaError_t launch_swiglu_tc(const void* x, int dt, int T, const uint32_t* row_map, const int32_t* row_off,
                             const int32_t* tile_off, int R, const moe_experts& ex, void* h,
                             void* xs16, int* status, cudaStream_t s, bool h_perm = false);
cudaError_t launch_down_tc(const void* h, const int32_t* row_off, const int32_t* tile_off, int R,
                           const moe_experts& ex, void* ys, int* status, cudaStream_t s,
                           bool h_perm = false);

// The decode layer fused into one cooperative launch (q4 experts, bf16 or
// fp16 activations, T <= 32, T*k <= 256, E <= 256, d and F multiples of 128 and at
// most 2048). Writes the same workspace tables as the separate stages (logits,
// top-k, sort tables, x16, h, ys in fp16) and y; `sync` is a 4-byte scratch
// word.
bool decode_fused_ok(int T, int k, int E, int d, int F, int fmt, int dt);
cudaError_t launch_decode_fused(const void* x, int dt, const void* w_router, const float* bias,
                                const moe_experts& ex, int T, int k, int BM, float* logits,
                                int32_t* idx, float* w, uint32_t* order, uint32_t* inv_order,
                                uint32_t* row_map, int32_t* counts, int32_t* row_off,
                                int32_t* tile_off, void* x16, void* h, void* ys, void* y,
                                unsigned* sync, int* status, cudaStream_t s);

cudaError_t launch_combine(const void* ys, const uint32_t* inv_order, const float* w, int T, int k,
                           int d, int dt, void* y, cudaStream_t s);

}  // namespace moe
