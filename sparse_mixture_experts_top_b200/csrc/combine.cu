// Score-weighted unsort back to token order.
//
// DS4Server issue #112, "Current upstream route": _scatter_unsort(y,
// inv_order, ...); mlxcel PR #275, "What it does": out = sum_k scores[k] *
// down_k(...). The pages' plan ("5.5 real sparse MoE kernels (Metal)",
// Scope -- in) adds the expert outputs with threadgroup atomics; here each
// output element is owned by one thread, which gathers its k rows through
// inv_order and sums them in j order -- no atomics, deterministic.
#include <type_traits>

#include "common.cuh"
#include "launch.h"

namespace moe {

// One thread per 8 consecutive outputs of one token: k gathers of 8 ys values
// (fp16 for 16-bit activations, fp32 for fp32), fp32 fused multiply-adds in j
// order, one rounding to TA.
template <typename TA, typename TY>
__global__ void __launch_bounds__(256) combine_kernel(const TY* __restrict__ ys,
                                                      const uint32_t* __restrict__ inv_order,
                                                      const float* __restrict__ w, int T, int k,
                                                      int d, TA* __restrict__ y) {
  pdl_wait();
  pdl_launch();
  constexpr int V = 8;
  const int per_row = d / V;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= (long long)T * per_row) return;
  const int t = (int)(gid / per_row);
  const int o = (int)(gid % per_row) * V;
  float acc[V];
#pragma unroll
  for (int i = 0; i < V; ++i) acc[i] = 0.f;
  for (int j = 0; j < k; ++j) {
    const float wj = __ldg(w + (size_t)t * k + j);
    const TY* src = ys + (size_t)__ldg(inv_order + (size_t)t * k + j) * d + o;
    float v[8];
    if constexpr (sizeof(TY) == 2) {
      const uint4 a = *reinterpret_cast<const uint4*>(src);
      const uint32_t u[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[i]));
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
      }
    } else {
      const float4 a = *reinterpret_cast<const float4*>(src);
      const float4 b = *reinterpret_cast<const float4*>(src + 4);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
      v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = fmaf(wj, v[i], acc[i]);
  }
  TA* dst = y + (size_t)t * d + o;
  if constexpr (sizeof(TA) == 2) {
    constexpr bool kF16 = std::is_same<TA, __half>::value;
    uint4 out;
    out.x = kF16 ? pack_f16x2(acc[0], acc[1]) : pack_bf16x2(acc[0], acc[1]);
    out.y = kF16 ? pack_f16x2(acc[2], acc[3]) : pack_bf16x2(acc[2], acc[3]);
    out.z = kF16 ? pack_f16x2(acc[4], acc[5]) : pack_bf16x2(acc[4], acc[5]);
    out.w = kF16 ? pack_f16x2(acc[6], acc[7]) : pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(dst) = out;
  } else {
    *reinterpret_cast<float4*>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    *reinterpret_cast<float4*>(dst + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

cudaError_t launch_combine(const void* ys, const uint32_t* inv_order, const float* w, int T, int k,
                           int d, int dt, void* y, cudaStream_t s) {
  const long long n = (long long)T * (d / 8);
  if (n == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((n + 255) / 256);
  if (dt == MOE_BF16)
    launch_pdl(combine_kernel<__nv_bfloat16, __half>, blocks, 256, 0, s, (const __half*)ys,
               inv_order, w, T, k, d, (__nv_bfloat16*)y);
  else if (dt == MOE_F16)
    launch_pdl(combine_kernel<__half, __half>, blocks, 256, 0, s, (const __half*)ys, inv_order, w,
               T, k, d, (__half*)y);
  else
    launch_pdl(combine_kernel<float, float>, blocks, 256, 0, s, (const float*)ys, inv_order, w, T,
               k, d, (float*)y);
  return cudaGetLastError();
}

}  // namespace moe
