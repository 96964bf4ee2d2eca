// Weight-streaming grouped expert kernels (the decode regime).
//
// mlx-lm PR #2044, "What": for T = 1 gate and up are computed in one GEMV
// pass and the down projection runs over (slot, row block) so all k experts
// are in flight; for T > 1 slots are grouped by expert so each expert's
// weights are read and dequantised once per tile instead of once per
// (token, slot). mlxcel PR #275, "What it does": in-kernel affine dequant-GEMV
// of gate/up, swiglu, dequant-GEMV of down.
//
// One warp owns one output feature of one tile (<= BM sorted rows of one
// expert, found from tile_off by binary search): it streams that weight row
// (gate and up rows together for the SwiGLU kernel) once with 16-byte loads,
// dequantises in registers, and accumulates all the tile's token rows in
// fp32, then warp-reduces. Every selected expert's bytes are read once per
// call when BM covers the expert's rows.
#include <cuda_fp16.h>

#include <type_traits>

#include "common.cuh"
#include "launch.h"

namespace moe {

// ------------------------------------------------------------ weight words

// A 32-bit word of a weight row decoded to EPW floats.
template <int FMT> struct WDecode;

template <> struct WDecode<MOE_W_F32> {
  static constexpr int EPW = 1;
  __device__ __forceinline__ static void run(uint32_t w, float s, float b, float* out) {
    out[0] = __uint_as_float(w);
  }
};
template <> struct WDecode<MOE_W_BF16> {
  static constexpr int EPW = 2;
  __device__ __forceinline__ static void run(uint32_t w, float s, float b, float* out) {
    float2 v = bf16x2_to_f32x2(w);
    out[0] = v.x;
    out[1] = v.y;
  }
};
template <> struct WDecode<MOE_W_Q4G64> {
  static constexpr int EPW = 8;
  // value = scale * q + bias, q = bits [4j, 4j+3] of the word (element j)
  __device__ __forceinline__ static void run(uint32_t w, float s, float b, float* out) {
#pragma unroll
    for (int j = 0; j < 8; ++j) out[j] = fmaf(s, (float)((w >> (4 * j)) & 0xFu), b);
  }
};

// The hidden rows h between the two projections: fp16 for bf16 activations
// (the tensor-core operand format, 11-bit precision), fp32 for fp32.
template <typename TA> struct HType { using T = float; };
template <> struct HType<__nv_bfloat16> { using T = __half; };

__device__ __forceinline__ float2 f16x2_to_f32x2(uint32_t v) {
  return __half22float2(*reinterpret_cast<const __half2*>(&v));
}

// N consecutive activations starting at p (16-, 8- or 4-byte aligned) as floats.
template <typename TA, int N>
__device__ __forceinline__ void load_act(const TA* p, float* out) {
  if constexpr (std::is_same<TA, __half>::value) {
    static_assert(N == 2 || N == 8, "fp16 rows come in words of 2 or 8");
    if constexpr (N == 8) {
      uint4 v = ldg_v4(p);
      float2 a = f16x2_to_f32x2(v.x), b = f16x2_to_f32x2(v.y);
      float2 c = f16x2_to_f32x2(v.z), d = f16x2_to_f32x2(v.w);
      out[0] = a.x; out[1] = a.y; out[2] = b.x; out[3] = b.y;
      out[4] = c.x; out[5] = c.y; out[6] = d.x; out[7] = d.y;
    } else {
      float2 a = f16x2_to_f32x2(*reinterpret_cast<const uint32_t*>(p));
      out[0] = a.x; out[1] = a.y;
    }
  } else if constexpr (sizeof(TA) == 2) {
    static_assert(N == 2 || N == 8, "bf16 activations come in words of 2 or 8");
    if constexpr (N == 8) {
      uint4 v = ldg_v4(p);
      float2 a = bf16x2_to_f32x2(v.x), b = bf16x2_to_f32x2(v.y);
      float2 c = bf16x2_to_f32x2(v.z), d = bf16x2_to_f32x2(v.w);
      out[0] = a.x; out[1] = a.y; out[2] = b.x; out[3] = b.y;
      out[4] = c.x; out[5] = c.y; out[6] = d.x; out[7] = d.y;
    } else {
      float2 a = bf16x2_to_f32x2(*reinterpret_cast<const uint32_t*>(p));
      out[0] = a.x; out[1] = a.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) out[i] = p[i];
  }
}

// Elements of the weight row covered by 32-bit word `wi` start at wi*EPW.
// q4 scales/biases: one per 64 elements.
template <int FMT>
__device__ __forceinline__ void scale_bias(const uint16_t* s, const uint16_t* b, size_t row,
                                           int K, int elem, float& sv, float& bv) {
  if constexpr (FMT == MOE_W_Q4G64) {
    size_t g = row * (size_t)(K / 64) + elem / 64;
    sv = bf16_bits_to_f32(__ldg(s + g));
    bv = bf16_bits_to_f32(__ldg(b + g));
  } else {
    sv = 1.f;
    bv = 0.f;
  }
}

constexpr int kRowsPerPass = 8;   // token rows accumulated per pass over a weight row
constexpr int kWarpsPerBlock = 8;

// ------------------------------------------------------------ gate|up

template <typename TA, int FMT>
__global__ void __launch_bounds__(256) swiglu_gemv_kernel(
    const TA* __restrict__ x, const uint32_t* __restrict__ row_map,
    const int32_t* __restrict__ row_off, const int32_t* __restrict__ tile_off, int BM, int E, int d,
    int F, const uint32_t* __restrict__ wgu, const uint16_t* __restrict__ sgu,
    const uint16_t* __restrict__ bgu, typename HType<TA>::T* __restrict__ h, int* status) {
  using TH = typename HType<TA>::T;
  using D = WDecode<FMT>;
  constexpr int EPW = D::EPW;
  const int tau = blockIdx.y;
  if (tau >= __ldg(tile_off + E)) return;
  const int e = expert_of_tile(tile_off, E, tau);
  const int r0 = __ldg(row_off + e) + (tau - __ldg(tile_off + e)) * BM;
  const int r1 = min(__ldg(row_off + e + 1), r0 + BM);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int f = blockIdx.x * kWarpsPerBlock + warp;
  if (f >= F) return;

  const int words = d / EPW;                               // 32-bit words per weight row
  const size_t grow = (size_t)e * 2 * F + f;               // gate row
  const size_t urow = grow + F;                            // up row
  const uint32_t* gp = wgu + grow * words;
  const uint32_t* up = wgu + urow * words;

  for (int rb = r0; rb < r1; rb += kRowsPerPass) {
    const int nr = min(kRowsPerPass, r1 - rb);
    const TA* xr[kRowsPerPass];
#pragma unroll
    for (int j = 0; j < kRowsPerPass; ++j) xr[j] = x + (size_t)row_map[rb + (j < nr ? j : 0)] * d;
    float ag[kRowsPerPass], au[kRowsPerPass];
#pragma unroll
    for (int j = 0; j < kRowsPerPass; ++j) ag[j] = au[j] = 0.f;
    // each lane takes 16-byte chunks (4 words) lane, lane + 32, ...
    for (int c = lane; c * 4 < words; c += 32) {
      uint4 gw = ldg_nc_v4(gp + c * 4);
      uint4 uw = ldg_nc_v4(up + c * 4);
      const uint32_t gws[4] = {gw.x, gw.y, gw.z, gw.w};
      const uint32_t uws[4] = {uw.x, uw.y, uw.z, uw.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int elem = (c * 4 + q) * EPW;
        float gs, gb, us, ub;
        scale_bias<FMT>(sgu, bgu, grow, d, elem, gs, gb);
        scale_bias<FMT>(sgu, bgu, urow, d, elem, us, ub);
        float gv[EPW], uv[EPW];
        D::run(gws[q], gs, gb, gv);
        D::run(uws[q], us, ub, uv);
#pragma unroll
        for (int j = 0; j < kRowsPerPass; ++j) {
          if (j < nr) {
            float xv[EPW];
            load_act<TA, EPW>(xr[j] + elem, xv);
#pragma unroll
            for (int i = 0; i < EPW; ++i) {
              ag[j] = fmaf(xv[i], gv[i], ag[j]);
              au[j] = fmaf(xv[i], uv[i], au[j]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kRowsPerPass; ++j) {
      const float g = warp_sum(ag[j]);
      const float u = warp_sum(au[j]);
      if (lane == 0 && j < nr) {
        const float v = swiglu(g, u);
        if constexpr (std::is_same<TH, __half>::value) {
          if (!(fabsf(v) < 65520.f)) report_status(status, MOE_ERR_RANGE);
          h[(size_t)(rb + j) * F + f] = __float2half_rn(v);
        } else {
          h[(size_t)(rb + j) * F + f] = v;
        }
      }
    }
  }
}

// ------------------------------------------------------------ down

template <typename TA, int FMT>
__global__ void __launch_bounds__(256) down_gemv_kernel(
    const typename HType<TA>::T* __restrict__ hin, const int32_t* __restrict__ row_off,
    const int32_t* __restrict__ tile_off, int BM, int E, int d, int F,
    const uint32_t* __restrict__ wdn, const uint16_t* __restrict__ sdn,
    const uint16_t* __restrict__ bdn, float* __restrict__ ys) {
  using D = WDecode<FMT>;
  constexpr int EPW = D::EPW;
  const int tau = blockIdx.y;
  if (tau >= __ldg(tile_off + E)) return;
  const int e = expert_of_tile(tile_off, E, tau);
  const int r0 = __ldg(row_off + e) + (tau - __ldg(tile_off + e)) * BM;
  const int r1 = min(__ldg(row_off + e + 1), r0 + BM);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int o = blockIdx.x * kWarpsPerBlock + warp;
  if (o >= d) return;

  const int words = F / EPW;
  const size_t wrow = (size_t)e * d + o;
  const uint32_t* wp = wdn + wrow * words;
  for (int rb = r0; rb < r1; rb += kRowsPerPass) {
    const int nr = min(kRowsPerPass, r1 - rb);
    float acc[kRowsPerPass];
#pragma unroll
    for (int j = 0; j < kRowsPerPass; ++j) acc[j] = 0.f;
    for (int c = lane; c * 4 < words; c += 32) {
      uint4 ww = ldg_nc_v4(wp + c * 4);
      const uint32_t wws[4] = {ww.x, ww.y, ww.z, ww.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int elem = (c * 4 + q) * EPW;
        float s, b;
        scale_bias<FMT>(sdn, bdn, wrow, F, elem, s, b);
        float wv[EPW];
        D::run(wws[q], s, b, wv);
#pragma unroll
        for (int j = 0; j < kRowsPerPass; ++j) {
          if (j < nr) {
            float hv[EPW];
            load_act<typename HType<TA>::T, EPW>(hin + (size_t)(rb + j) * F + elem, hv);
#pragma unroll
            for (int i = 0; i < EPW; ++i) acc[j] = fmaf(hv[i], wv[i], acc[j]);
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kRowsPerPass; ++j) {
      const float v = warp_sum(acc[j]);
      if (lane == 0 && j < nr) ys[(size_t)(rb + j) * d + o] = v;
    }
  }
}

// ------------------------------------------------------------ launchers

cudaError_t launch_swiglu_gemv(const void* x, int dt, const uint32_t* row_map,
                               const int32_t* row_off, const int32_t* tile_off, int BM, int R,
                               const moe_experts& ex, void* h, int* status, cudaStream_t s) {
  const long long tiles = max_tiles(R, ex.E, BM);
  if (tiles <= 0) return cudaSuccess;
  if (tiles > 65535) return cudaErrorInvalidConfiguration;
  dim3 grid((ex.F + kWarpsPerBlock - 1) / kWarpsPerBlock, (unsigned)tiles);
  const uint32_t* w = (const uint32_t*)ex.w_gu;
  const uint16_t* sc = (const uint16_t*)ex.s_gu;
  const uint16_t* bi = (const uint16_t*)ex.b_gu;
#define MOE_SWIGLU(TA, FMT)                                                                    \
  swiglu_gemv_kernel<TA, FMT><<<grid, 256, 0, s>>>((const TA*)x, row_map, row_off, tile_off, BM, \
                                                   ex.E, ex.d, ex.F, w, sc, bi,                  \
                                                   (typename HType<TA>::T*)h, status)
  if (dt == MOE_F32 && ex.fmt == MOE_W_F32) MOE_SWIGLU(float, MOE_W_F32);
  else if (dt == MOE_BF16 && ex.fmt == MOE_W_BF16) MOE_SWIGLU(__nv_bfloat16, MOE_W_BF16);
  else if (dt == MOE_BF16 && ex.fmt == MOE_W_Q4G64) MOE_SWIGLU(__nv_bfloat16, MOE_W_Q4G64);
  else return cudaErrorInvalidValue;
#undef MOE_SWIGLU
  return cudaGetLastError();
}

cudaError_t launch_down_gemv(const void* h, int dt, const int32_t* row_off,
                             const int32_t* tile_off, int BM, int R, const moe_experts& ex,
                             void* ys, cudaStream_t s) {
  const long long tiles = max_tiles(R, ex.E, BM);
  if (tiles <= 0) return cudaSuccess;
  if (tiles > 65535) return cudaErrorInvalidConfiguration;
  dim3 grid((ex.d + kWarpsPerBlock - 1) / kWarpsPerBlock, (unsigned)tiles);
  const uint32_t* w = (const uint32_t*)ex.w_dn;
  const uint16_t* sc = (const uint16_t*)ex.s_dn;
  const uint16_t* bi = (const uint16_t*)ex.b_dn;
#define MOE_DOWN(TA, FMT)                                                                    \
  down_gemv_kernel<TA, FMT><<<grid, 256, 0, s>>>((const typename HType<TA>::T*)h, row_off,    \
                                                 tile_off, BM, ex.E, ex.d, ex.F, w, sc, bi,     \
                                                 (float*)ys)
  if (dt == MOE_F32 && ex.fmt == MOE_W_F32) MOE_DOWN(float, MOE_W_F32);
  else if (dt == MOE_BF16 && ex.fmt == MOE_W_BF16) MOE_DOWN(__nv_bfloat16, MOE_W_BF16);
  else if (dt == MOE_BF16 && ex.fmt == MOE_W_Q4G64) MOE_DOWN(__nv_bfloat16, MOE_W_Q4G64);
  else return cudaErrorInvalidValue;
#undef MOE_DOWN
  return cudaGetLastError();
}

}  // namespace moe
