// Shared device helpers of the MoE forward kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

constexpr int kWarp = 32;

// ---------------------------------------------------------------- numbers

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h16) {
  return __uint_as_float(h16 << 16);
}

// (lo, hi) halves of a packed bf16 pair as floats
__device__ __forceinline__ float2 bf16x2_to_f32x2(uint32_t v) {
  return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xFFFF0000u));
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return (uint32_t)f32_to_bf16_bits(lo) | ((uint32_t)f32_to_bf16_bits(hi) << 16);
}

template <typename T> struct Act;
template <> struct Act<float> {
  static __device__ __forceinline__ float load(const float* p, size_t i) { return p[i]; }
  static __device__ __forceinline__ void store(float* p, size_t i, float v) { p[i] = v; }
};
template <> struct Act<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16* p, size_t i) {
    return __bfloat162float(p[i]);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, size_t i, float v) {
    p[i] = __float2bfloat16_rn(v);
  }
};
template <> struct Act<__half> {
  static __device__ __forceinline__ float load(const __half* p, size_t i) {
    return __half2float(p[i]);
  }
  static __device__ __forceinline__ void store(__half* p, size_t i, float v) {
    p[i] = __float2half_rn(v);
  }
};

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// silu(g) * u with silu(g) = g * sigmoid(g) = g / (1 + exp(-g)); the fast
// division (2 ulp; 0 once 1 + exp(-g) passes 2^126, i.e. silu below 1e-36 in
// magnitude) costs far less than the IEEE one and stays far below the
// rounding of h to its storage type
__device__ __forceinline__ float swiglu(float g, float u) {
  return __fdividef(g, 1.0f + __expf(-g)) * u;
}

// act(g) * u for the GLU's gate activation (moe_act): silu, or the tanh form
// of GELU, 0.5 g (1 + tanh(sqrt(2/pi) (g + 0.044715 g^3)))
__device__ __forceinline__ float glu(int act, float g, float u) {
  if (act == MOE_ACT_GEGLU_TANH) {
    const float z = 0.7978845608028654f * fmaf(0.044715f * g, g * g, g);
    return 0.5f * g * (1.0f + tanhf(z)) * u;
  }
  return swiglu(g, u);
}

// Elements per scale and bias of a 4-bit format (moe_wfmt), 0 for the others
__host__ __device__ constexpr int q4_group(int fmt) {
  return fmt == MOE_W_Q4G64 ? 64 : fmt == MOE_W_Q4G32 ? 32 : fmt == MOE_W_Q4G128 ? 128 : 0;
}

// Elements per scale and bias of any quantised format (4- or 8-bit), 0 else
__host__ __device__ constexpr int wq_group(int fmt) {
  return fmt == MOE_W_Q8G64 ? 64 : q4_group(fmt);
}

// ---------------------------------------------------------------- warps

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ uint32_t lane_id() {
  uint32_t l;
  asm volatile("mov.u32 %0, %%laneid;" : "=r"(l));
  return l;
}

// ---------------------------------------------------------------- loads

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint4 ldg_v4(const void* p) {
  return *reinterpret_cast<const uint4*>(p);
}

// ---------------------------------------------------------------- tiles

// Expert of tile tau: the largest e with tile_off[e] <= tau (empty experts
// have tile_off[e] == tile_off[e+1] and are skipped by taking the largest).
__device__ __forceinline__ int expert_of_tile(const int32_t* tile_off, int E, int tau) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(tile_off + mid) <= tau) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ---------------------------------------------------------------- launches

// Programmatic dependent launch. Every kernel of the library waits, before
// it reads anything an earlier kernel in the stream wrote, until those
// kernels have completed and their memory is visible (griddepcontrol.wait),
// then lets the next kernel be scheduled (launch_dependents); launches carry
// the programmatic-serialization attribute, so a kernel's launch and prologue
// overlap the tail of the one before it.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// The same search by one warp in two dependent loads (E <= 1024): the lanes
// first read every ceil(E/32)-th entry, then the entries of the segment the
// first round picked. All lanes return the same expert.
__device__ __forceinline__ int expert_of_tile_warp(const int32_t* tile_off, int E, int tau) {
  const int lane = threadIdx.x & 31;
  const int stride = (E + 31) >> 5;
  const int i0 = lane * stride;
  const bool ok0 = i0 < E && __ldg(tile_off + i0) <= tau;
  const unsigned m0 = __ballot_sync(0xffffffffu, ok0);   // lane 0 always qualifies
  const int base = (31 - __clz(m0)) * stride;
  const int i1 = base + lane;
  const bool ok1 = lane < stride && i1 < E && __ldg(tile_off + i1) <= tau;
  const unsigned m1 = __ballot_sync(0xffffffffu, ok1);
  return base + (31 - __clz(m1));
}

// ---------------------------------------------------------------- status

// Record the first device-side error in the status word `st` (a device
// pointer the host obtains for the library's status symbol).
__device__ __forceinline__ void report_status(int* st, int code) {
  if (st) atomicCAS(st, 0, code);
}

}  // namespace moe
