// Router: logits x . W_r + b, then softmax / top-k / renormalise.
//
// "5.5 real sparse MoE kernels (Metal)", Scope -- in: a top-K routing kernel
// from routing logits to (top_k_indices, top_k_weights) with no host round
// trip; MOE_OPTIMIZATION_COMPLETE.md, "Mega Kernel Architecture": router
// matmul, softmax and top-K on the GPU.
//
// Top-k runs one warp per token: every lane holds E/32 logits in registers
// with their orderable 32-bit keys; per round a warp max-reduce of the lanes'
// best keys and a min-reduce of the expert indices holding that key give the
// best remaining expert with the lowest index among equal values; k rounds of
// that select the experts best first. -0.0 is mapped to +0.0 and NaN to the
// lowest key, so the order is total and deterministic.
#include "common.cuh"
#include "launch.h"

namespace moe {

// ------------------------------------------------------------ logits (SIMT)

// Few tokens: one warp per (expert, group of up to 8 tokens), 16-byte loads
// along d, warp reduction at the end.
template <typename T>
__global__ void __launch_bounds__(256) router_gemv_kernel(const T* __restrict__ x,
                                                          const T* __restrict__ wr,
                                                          const float* __restrict__ bias, int Tn,
                                                          int d, int E, float* __restrict__ out) {
  pdl_wait();
  pdl_launch();
  constexpr int TG = 8;                         // tokens per warp
  constexpr int VE = 16 / sizeof(T);            // elements per 16-byte load
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int ngroups = (Tn + TG - 1) / TG;
  if (warp >= E * ngroups) return;
  const int e = warp % E;
  const int t0 = (warp / E) * TG;
  const int nt = min(TG, Tn - t0);
  float acc[TG];
#pragma unroll
  for (int j = 0; j < TG; ++j) acc[j] = 0.f;
  const T* wrow = wr + (size_t)e * d;
  for (int c = lane * VE; c < d; c += 32 * VE) {
    float wv[VE];
    uint4 wraw = ldg_v4(wrow + c);
    const T* wp = reinterpret_cast<const T*>(&wraw);
#pragma unroll
    for (int q = 0; q < VE; ++q) wv[q] = Act<T>::load(wp, q);
#pragma unroll
    for (int j = 0; j < TG; ++j) {
      if (j < nt) {
        uint4 xraw = ldg_v4(x + (size_t)(t0 + j) * d + c);
        const T* xp = reinterpret_cast<const T*>(&xraw);
#pragma unroll
        for (int q = 0; q < VE; ++q) acc[j] = fmaf(Act<T>::load(xp, q), wv[q], acc[j]);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < TG; ++j) {
    float v = warp_sum(acc[j]);
    if (lane == 0 && j < nt) out[(size_t)(t0 + j) * E + e] = v + (bias ? bias[e] : 0.f);
  }
}

// Many tokens: 64 x 64 output tile per 256-thread block, 4 x 4 per thread,
// operands staged through shared memory as fp32 in k-major order.
template <typename T>
__global__ void __launch_bounds__(256) router_tile_kernel(const T* __restrict__ x,
                                                          const T* __restrict__ wr,
                                                          const float* __restrict__ bias, int Tn,
                                                          int d, int E, float* __restrict__ out) {
  pdl_wait();
  pdl_launch();
  constexpr int BT = 64, BE = 64, BK = 32;
  __shared__ float As[BK][BT + 4];
  __shared__ float Bs[BK][BE + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int t0 = blockIdx.y * BT, e0 = blockIdx.x * BE;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < d; k0 += BK) {
    for (int i = tid; i < BT * BK; i += 256) {
      int r = i / BK, c = i % BK;
      int t = t0 + r, e = e0 + r;
      As[c][r] = (t < Tn) ? Act<T>::load(x, (size_t)t * d + k0 + c) : 0.f;
      Bs[c][r] = (e < E) ? Act<T>::load(wr, (size_t)e * d + k0 + c) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < BK; ++c) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[c][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[c][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int t = t0 + ty * 4 + i;
    if (t >= Tn) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int e = e0 + tx * 4 + j;
      if (e < E) out[(size_t)t * E + e] = acc[i][j] + (bias ? bias[e] : 0.f);
    }
  }
}

cudaError_t launch_router_logits(const void* x, int dt, const void* w_router, const float* bias,
                                 int T, int d, int E, float* logits, cudaStream_t s) {
  if (T <= 64) {
    int warps = E * ((T + 7) / 8);
    int blocks = (warps * 32 + 255) / 256;
    if (dt == MOE_BF16)
      launch_pdl(router_gemv_kernel<__nv_bfloat16>, blocks, 256, 0, s, 
          (const __nv_bfloat16*)x, (const __nv_bfloat16*)w_router, bias, T, d, E, logits);
    else if (dt == MOE_F16)
      launch_pdl(router_gemv_kernel<__half>, blocks, 256, 0, s, (const __half*)x,
                 (const __half*)w_router, bias, T, d, E, logits);
    else
      launch_pdl(router_gemv_kernel<float>, blocks, 256, 0, s, (const float*)x, (const float*)w_router,
                                                       bias, T, d, E, logits);
  } else {
    dim3 grid((E + 63) / 64, (T + 63) / 64);
    if (dt == MOE_BF16)
      launch_pdl(router_tile_kernel<__nv_bfloat16>, grid, 256, 0, s, 
          (const __nv_bfloat16*)x, (const __nv_bfloat16*)w_router, bias, T, d, E, logits);
    else if (dt == MOE_F16)
      launch_pdl(router_tile_kernel<__half>, grid, 256, 0, s, (const __half*)x,
                 (const __half*)w_router, bias, T, d, E, logits);
    else
      launch_pdl(router_tile_kernel<float>, grid, 256, 0, s, (const float*)x, (const float*)w_router,
                                                     bias, T, d, E, logits);
  }
  return cudaGetLastError();
}

// ------------------------------------------------------------ top-k

// Orderable 32-bit image of a float: larger float -> larger key; -0 -> +0;
// NaN -> 0 (below -inf, whose key is 0x007FFFFF).
__device__ __forceinline__ uint32_t order_key(float v) {
  if (v == 0.0f) v = 0.0f;
  uint32_t u = __float_as_uint(v);
  if (isnan(v)) return 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// VPL = logits held per lane (E <= 32 * VPL). Each of the k rounds takes the
// lane's best remaining expert (largest key, the lowest index among equal
// keys), the warp maximum of those keys and then the lowest expert index among
// the lanes that hold it: two single-instruction warp reductions per selected
// expert instead of a five-step 64-bit shuffle tree.
template <int VPL>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits, int T, int E,
                                                   int k, int32_t* __restrict__ idx_out,
                                                   float* __restrict__ w_out) {
  pdl_wait();
  pdl_launch();
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  const float* row = logits + (size_t)t * E;
  uint32_t key[VPL];
  float val[VPL];
  uint32_t avail = 0;                 // bit i: expert lane + 32 i exists and is not taken
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane + 32 * i;
    val[i] = e < E ? row[e] : 0.f;
    key[i] = order_key(val[i]);
    if (e < E) avail |= 1u << i;
  }
  int my_e = 0;                       // lane j keeps the j-th selected expert and its logit
  float my_v = 0.f;
  for (int j = 0; j < k; ++j) {
    uint32_t bk = 0;
    int bi = -1;
    float bv = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      if (((avail >> i) & 1u) && (bi < 0 || key[i] > bk)) {
        bk = key[i];
        bi = i;
        bv = val[i];
      }
    }
    const uint32_t M = __reduce_max_sync(0xffffffffu, bi >= 0 ? bk : 0u);
    const uint32_t ce = (bi >= 0 && bk == M) ? (uint32_t)(lane + 32 * bi) : 0xFFFFFFFFu;
    const uint32_t es = __reduce_min_sync(0xffffffffu, ce);
    const float v = __shfl_sync(0xffffffffu, bv, (int)(es & 31u));
    if ((int)(es & 31u) == lane) avail &= ~(1u << (es >> 5));
    if (lane == j) {
      my_e = (int)es;
      my_v = v;
    }
  }
  // weights: exp(L_j - m) / sum over the selected, m = the best logit
  const float m = __shfl_sync(0xffffffffu, my_v, 0);
  const float ex = lane < k ? __expf(my_v - m) : 0.f;
  const float den = warp_sum(ex);
  if (lane < k) {
    idx_out[(size_t)t * k + lane] = my_e;
    w_out[(size_t)t * k + lane] = ex / den;
  }
}

cudaError_t launch_topk(const float* logits, int T, int E, int k, int32_t* idx, float* w,
                        cudaStream_t s) {
  const int blocks = (T * 32 + 255) / 256;
  if (E <= 32) launch_pdl(topk_kernel<1>, blocks, 256, 0, s, logits, T, E, k, idx, w);
  else if (E <= 64) launch_pdl(topk_kernel<2>, blocks, 256, 0, s, logits, T, E, k, idx, w);
  else if (E <= 128) launch_pdl(topk_kernel<4>, blocks, 256, 0, s, logits, T, E, k, idx, w);
  else if (E <= 256) launch_pdl(topk_kernel<8>, blocks, 256, 0, s, logits, T, E, k, idx, w);
  else if (E <= 512) launch_pdl(topk_kernel<16>, blocks, 256, 0, s, logits, T, E, k, idx, w);
  else if (E <= 1024) launch_pdl(topk_kernel<32>, blocks, 256, 0, s, logits, T, E, k, idx, w);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace moe
