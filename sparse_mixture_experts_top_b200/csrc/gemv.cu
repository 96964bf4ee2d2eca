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

template <> struct WDecode<MOE_W_Q8G64> {
  static constexpr int EPW = 4;
  // value = scale * q + bias, q = byte j of the word (element j)
  __device__ __forceinline__ static void run(uint32_t w, float s, float b, float* out) {
#pragma unroll
    for (int j = 0; j < 4; ++j) out[j] = fmaf(s, (float)((w >> (8 * j)) & 0xFFu), b);
  }
};

// The hidden rows h between the two projections: fp16 for 16-bit activations
// (the tensor-core operand format, 11-bit precision), fp32 for fp32.
template <typename TA> struct HType { using T = float; };
template <> struct HType<__nv_bfloat16> { using T = __half; };
template <> struct HType<__half> { using T = __half; };

__device__ __forceinline__ float2 f16x2_to_f32x2(uint32_t v) {
  return __half22float2(*reinterpret_cast<const __half2*>(&v));
}

// N consecutive activations starting at p (16-, 8- or 4-byte aligned) as floats.
template <typename TA, int N>
__device__ __forceinline__ void load_act(const TA* p, float* out) {
  if constexpr (std::is_same<TA, __half>::value) {
    static_assert(N == 2 || N == 4 || N == 8, "fp16 rows come in words of 2, 4 or 8");
    if constexpr (N == 4) {
      uint2 v = *reinterpret_cast<const uint2*>(p);
      float2 a = f16x2_to_f32x2(v.x), b = f16x2_to_f32x2(v.y);
      out[0] = a.x; out[1] = a.y; out[2] = b.x; out[3] = b.y;
    } else if constexpr (N == 8) {
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
    static_assert(N == 2 || N == 4 || N == 8, "bf16 activations come in words of 2, 4 or 8");
    if constexpr (N == 4) {
      uint2 v = *reinterpret_cast<const uint2*>(p);
      float2 a = bf16x2_to_f32x2(v.x), b = bf16x2_to_f32x2(v.y);
      out[0] = a.x; out[1] = a.y; out[2] = b.x; out[3] = b.y;
    } else if constexpr (N == 8) {
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
// q4 scales/biases: one per gs (32, 64 or 128) elements; every 4-bit format
// runs the MOE_W_Q4G64 instantiation with its own gs.
template <int FMT>
__device__ __forceinline__ void scale_bias(const uint16_t* s, const uint16_t* b, size_t row,
                                           int K, int elem, int gs, float& sv, float& bv) {
  if constexpr (FMT == MOE_W_Q4G64 || FMT == MOE_W_Q8G64) {
    size_t g = row * (size_t)(K / gs) + elem / gs;
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
    const uint16_t* __restrict__ bgu, typename HType<TA>::T* __restrict__ h, int act, int qg,
    int* status) {
  pdl_wait();
  pdl_launch();
  using TH = typename HType<TA>::T;
  using D = WDecode<FMT>;
  constexpr int EPW = D::EPW;
  const int tau = blockIdx.y;
  if (tau >= __ldg(tile_off + E)) return;
  const int e = expert_of_tile_warp(tile_off, E, tau);
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
        scale_bias<FMT>(sgu, bgu, grow, d, elem, qg, gs, gb);
        scale_bias<FMT>(sgu, bgu, urow, d, elem, qg, us, ub);
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
        const float v = glu(act, g, u);
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
    const uint16_t* __restrict__ bdn, typename HType<TA>::T* __restrict__ ys, int qg,
    int* status) {
  pdl_wait();
  pdl_launch();
  using D = WDecode<FMT>;
  constexpr int EPW = D::EPW;
  const int tau = blockIdx.y;
  if (tau >= __ldg(tile_off + E)) return;
  const int e = expert_of_tile_warp(tile_off, E, tau);
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
        scale_bias<FMT>(sdn, bdn, wrow, F, elem, qg, s, b);
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
      if (lane == 0 && j < nr) {
        if (sizeof(typename HType<TA>::T) == 2) {
          // fp16 ys (16-bit activations): out-of-range values are reported
          if (!(fabsf(v) < 65520.f)) report_status(status, MOE_ERR_RANGE);
          reinterpret_cast<__half*>(ys)[(size_t)(rb + j) * d + o] = __float2half_rn(v);
        } else {
          reinterpret_cast<float*>(ys)[(size_t)(rb + j) * d + o] = v;
        }
      }
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
  launch_pdl(swiglu_gemv_kernel<TA, FMT>, grid, 256, 0, s, (const TA*)x, row_map, row_off, tile_off, BM, \
                                                   ex.E, ex.d, ex.F, w, sc, bi,                  \
                                                   (typename HType<TA>::T*)h, ex.act,          \
                                                   wq_group(ex.fmt), status)
  if (dt == MOE_F32 && ex.fmt == MOE_W_F32) MOE_SWIGLU(float, MOE_W_F32);
  else if (dt == MOE_BF16 && ex.fmt == MOE_W_BF16) MOE_SWIGLU(__nv_bfloat16, MOE_W_BF16);
  else if (dt == MOE_BF16 && q4_group(ex.fmt)) MOE_SWIGLU(__nv_bfloat16, MOE_W_Q4G64);
  else if (dt == MOE_BF16 && ex.fmt == MOE_W_Q8G64) MOE_SWIGLU(__nv_bfloat16, MOE_W_Q8G64);
  else if (dt == MOE_F16 && q4_group(ex.fmt)) MOE_SWIGLU(__half, MOE_W_Q4G64);
  else if (dt == MOE_F16 && ex.fmt == MOE_W_Q8G64) MOE_SWIGLU(__half, MOE_W_Q8G64);
  else return cudaErrorInvalidValue;
#undef MOE_SWIGLU
  return cudaGetLastError();
}

cudaError_t launch_down_gemv(const void* h, int dt, const int32_t* row_off,
                             const int32_t* tile_off, int BM, int R, const moe_experts& ex,
                             void* ys, int* status, cudaStream_t s) {
  const long long tiles = max_tiles(R, ex.E, BM);
  if (tiles <= 0) return cudaSuccess;
  if (tiles > 65535) return cudaErrorInvalidConfiguration;
  dim3 grid((ex.d + kWarpsPerBlock - 1) / kWarpsPerBlock, (unsigned)tiles);
  const uint32_t* w = (const uint32_t*)ex.w_dn;
  const uint16_t* sc = (const uint16_t*)ex.s_dn;
  const uint16_t* bi = (const uint16_t*)ex.b_dn;
#define MOE_DOWN(TA, FMT)                                                                    \
  launch_pdl(down_gemv_kernel<TA, FMT>, grid, 256, 0, s, (const typename HType<TA>::T*)h, row_off,    \
                                                 tile_off, BM, ex.E, ex.d, ex.F, w, sc, bi,     \
                                                 (typename HType<TA>::T*)ys,                \
                                                 wq_group(ex.fmt), status)
  // the down projection reads and writes fp16 for both 16-bit activation
  // types: one instantiation serves both
  const bool a16 = dt == MOE_BF16 || dt == MOE_F16;
  if (dt == MOE_F32 && ex.fmt == MOE_W_F32) MOE_DOWN(float, MOE_W_F32);
  else if (dt == MOE_BF16 && ex.fmt == MOE_W_BF16) MOE_DOWN(__nv_bfloat16, MOE_W_BF16);
  else if (a16 && q4_group(ex.fmt)) MOE_DOWN(__nv_bfloat16, MOE_W_Q4G64);
  else if (a16 && ex.fmt == MOE_W_Q8G64) MOE_DOWN(__nv_bfloat16, MOE_W_Q8G64);
  else return cudaErrorInvalidValue;
#undef MOE_DOWN
  return cudaGetLastError();
}


// ===================================================================
// q4 weights, 16-bit activations (fp16 operands): tensor-core GEMV (mma.sync m16n8k16, fp16
// operands, fp32 accumulate) for tiles of at most 16 token rows.
//
// A CTA of 4 warps owns one block of 16 weight rows of one tile -- for the
// gate|up projection rows g and g+8 of the block are gate row f0+g and up
// row f0+g, so SwiGLU happens in the lane that holds both accumulators; for
// the down projection they are output rows o0+g and o0+8+g. K is walked in
// steps of 128 elements, dealt round-robin to the 4 warps and reduced
// through shared memory at the end.
//
// In a step, lane (g = lane/4, c = lane%4) loads 16 bytes (32 nibbles,
// elements c*32 .. c*32+31 of the step) of each of its two rows, and the same
// 32 elements of its token row(s) from fp16 activations. Inside the 16-wide
// K slice of MMA m (m = 0..7) the element order is permuted identically for
// A and B: fragment columns (2c, 2c+1) and (2c+8, 2c+9) are elements
// c*32 + 4m + (0, 1) and c*32 + 4m + (2, 3). Those are consecutive nibbles of
// word m/2 and consecutive activations, so both fragments are contiguous
// loads and the dequantised pairs come out in fragment order.

constexpr int kMmaWarps = 4;
constexpr int kMmaMaxRows = 16;            // token rows per tile (two n8 groups)

__device__ __forceinline__ void mma_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t h2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t h2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t h2_from_bf16(uint32_t v16) {
  const float f = __uint_as_float(v16 << 16);
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %1;" : "=r"(d) : "f"(f));
  return d;
}
// nibbles of one word -> fp16 pairs (e0,e1) (e2,e3) (e4,e5) (e6,e7) of
// s*q + b, one rounding: q goes into the mantissa of fp16 1024.0 (exact),
// 1024 is subtracted exactly, one fused multiply-add applies scale and bias
__device__ __forceinline__ void q4_word_f16(uint32_t w, uint32_t s2, uint32_t b2, uint32_t* o) {
  const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
  const uint32_t p0 = __byte_perm(lo, hi, 0x5140), p1 = __byte_perm(lo, hi, 0x7362);
  const uint32_t M = 0x64646464u, c1024 = 0x64006400u;
  o[0] = h2_fma(h2_sub(__byte_perm(p0, M, 0x4140), c1024), s2, b2);
  o[1] = h2_fma(h2_sub(__byte_perm(p0, M, 0x4342), c1024), s2, b2);
  o[2] = h2_fma(h2_sub(__byte_perm(p1, M, 0x4140), c1024), s2, b2);
  o[3] = h2_fma(h2_sub(__byte_perm(p1, M, 0x4342), c1024), s2, b2);
}

// SWIGLU: x16 [T][d] fp16 activations through row_map, w = w_gu, out = h fp16
// else:   x16 = h [R][F] fp16 rows (contiguous), w = w_dn, out = ys fp32
template <bool SWIGLU>
__global__ void __launch_bounds__(kMmaWarps * 32) gemv_q4_mma_kernel(
    const __half* __restrict__ x16, const uint32_t* __restrict__ row_map,
    const int32_t* __restrict__ row_off, const int32_t* __restrict__ tile_off, int BM, int E,
    int d, int F, const uint32_t* __restrict__ w, const uint16_t* __restrict__ sc,
    const uint16_t* __restrict__ bi, void* __restrict__ out, int act, int gs, int* status) {
  pdl_wait();
  pdl_launch();
  __shared__ float red[kMmaWarps - 1][32][8];
  const int tau = blockIdx.y;
  if (tau >= __ldg(tile_off + E)) return;
  const int e = expert_of_tile_warp(tile_off, E, tau);
  const int r0 = __ldg(row_off + e) + (tau - __ldg(tile_off + e)) * BM;
  const int nv = min(__ldg(row_off + e + 1), r0 + BM) - r0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int K = SWIGLU ? d : F;                 // reduction length
  const int rows_e = SWIGLU ? 2 * F : d;        // weight rows per expert
  const int blk = blockIdx.x;                   // block of 16 weight rows
  const size_t row_lo = (size_t)e * rows_e + (SWIGLU ? blk * 8 + g : blk * 16 + g);
  const size_t row_hi = SWIGLU ? row_lo + F : row_lo + 8;
  const int words = K / 8, G = K / gs;         // gs: elements per scale (32, 64 or 128)
  const uint32_t* wlo = w + row_lo * words;
  const uint32_t* whi = w + row_hi * words;
  // token rows of this lane's B fragment: tokens g (group 0) and 8+g (group 1)
  const __half* xr[2];
  bool tok_ok[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int n = t * 8 + g;
    tok_ok[t] = n < nv;
    const size_t row = tok_ok[t] ? (SWIGLU ? (size_t)__ldg(row_map + r0 + n) : (size_t)(r0 + n)) : 0;
    xr[t] = x16 + row * K;
  }
  const bool two = nv > 8;
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  const int nsteps = K / 128;

  // one step's operands: this lane's 32 elements of both rows, their group's
  // scales and biases, and the same 32 activations of its two token rows
  struct Step {
    uint4 wl, wh;
    uint16_t sl, bl, sh, bh;
    uint4 xv[2][4];
  };
  auto load = [&](Step& S, int st) {
    const int k0 = st * 128 + c * 32;
    S.wl = ldg_nc_v4(wlo + k0 / 8);
    S.wh = ldg_nc_v4(whi + k0 / 8);
    const int grp = k0 / gs;                    // a lane's 32 elements share one group
    S.sl = __ldg(sc + row_lo * G + grp);
    S.bl = __ldg(bi + row_lo * G + grp);
    S.sh = __ldg(sc + row_hi * G + grp);
    S.bh = __ldg(bi + row_hi * G + grp);
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int q = 0; q < 4; ++q)
        S.xv[t][q] = (tok_ok[t] && (t == 0 || two)) ? ldg_v4(xr[t] + k0 + q * 8)
                                                    : make_uint4(0, 0, 0, 0);
  };
  auto compute = [&](const Step& S) {
    const uint32_t sl = h2_from_bf16(S.sl), bl = h2_from_bf16(S.bl);
    const uint32_t sh = h2_from_bf16(S.sh), bh = h2_from_bf16(S.bh);
    const uint32_t wlw[4] = {S.wl.x, S.wl.y, S.wl.z, S.wl.w};
    const uint32_t whw[4] = {S.wh.x, S.wh.y, S.wh.z, S.wh.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {               // word q: MMAs m = 2q, 2q+1
      uint32_t dl[4], dh[4];
      q4_word_f16(wlw[q], sl, bl, dl);
      q4_word_f16(whw[q], sh, bh, dh);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const uint32_t a[4] = {dl[2 * half], dh[2 * half], dl[2 * half + 1], dh[2 * half + 1]};
        // activations c*32 + 4m + (0..3) with m = 2q + half: uint32 words
        // 2m and 2m+1 of this lane's 64 bytes
        const int m = 2 * q + half;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (t == 1 && !two) break;
          const uint4 v = S.xv[t][m >> 1];
          mma_16816(acc[t], a, (m & 1) ? v.z : v.x, (m & 1) ? v.w : v.y);
        }
      }
    }
  };
  // steps warp, warp + 4, ...: the next step's loads are in flight while the
  // current one is dequantised and multiplied (two register buffers used in
  // turn -- never copied into each other, which would wait for the loads)
  Step b0, b1;
  int st = warp;
  if (st < nsteps) load(b0, st);
  while (st < nsteps) {
    if (st + kMmaWarps < nsteps) load(b1, st + kMmaWarps);
    compute(b0);
    st += kMmaWarps;
    if (st >= nsteps) break;
    if (st + kMmaWarps < nsteps) load(b0, st + kMmaWarps);
    compute(b1);
    st += kMmaWarps;
  }
  // reduce the 4 warps' partial sums (warp 0 keeps the result)
  if (warp > 0) {
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int i = 0; i < 4; ++i) red[warp - 1][lane][t * 4 + i] = acc[t][i];
  }
  __syncthreads();
  if (warp != 0) return;
#pragma unroll
  for (int wv = 0; wv < kMmaWarps - 1; ++wv)
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[t][i] += red[wv][lane][t * 4 + i];
  // lane (g, c) holds rows g and g+8 for tokens t*8 + 2c and t*8 + 2c + 1
#pragma unroll
  for (int t = 0; t < 2; ++t) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int n = t * 8 + 2 * c + j;
      if (n >= nv) continue;
      if (SWIGLU) {
        const float v = glu(act, acc[t][j], acc[t][2 + j]);
        if (!(fabsf(v) < 65520.f)) report_status(status, MOE_ERR_RANGE);
        reinterpret_cast<__half*>(out)[(size_t)(r0 + n) * F + blk * 8 + g] = __float2half_rn(v);
      } else {
        // fp16 ys; out-of-range values are reported
        const float v0 = acc[t][j], v1 = acc[t][2 + j];
        if (!(fabsf(v0) < 65520.f && fabsf(v1) < 65520.f)) report_status(status, MOE_ERR_RANGE);
        __half* ys = reinterpret_cast<__half*>(out);
        ys[(size_t)(r0 + n) * d + blk * 16 + g] = __float2half_rn(v0);
        ys[(size_t)(r0 + n) * d + blk * 16 + 8 + g] = __float2half_rn(v1);
      }
    }
  }
}

bool gemv_q4_mma_ok(const moe_experts& ex, int dt, int BM) {
  return q4_group(ex.fmt) != 0 && (dt == MOE_BF16 || dt == MOE_F16) && BM <= kMmaMaxRows && ex.d % 128 == 0 &&
         ex.F % 128 == 0;
}

cudaError_t launch_swiglu_q4_mma(const void* x16, const uint32_t* row_map, const int32_t* row_off,
                                 const int32_t* tile_off, int BM, int R, const moe_experts& ex,
                                 void* h, int* status, cudaStream_t s) {
  const long long tiles = max_tiles(R, ex.E, BM);
  if (tiles <= 0) return cudaSuccess;
  if (tiles > 65535) return cudaErrorInvalidConfiguration;
  dim3 grid(ex.F / 8, (unsigned)tiles);
  launch_pdl(gemv_q4_mma_kernel<true>, grid, kMmaWarps * 32, 0, s, 
      (const __half*)x16, row_map, row_off, tile_off, BM, ex.E, ex.d, ex.F,
      (const uint32_t*)ex.w_gu, (const uint16_t*)ex.s_gu, (const uint16_t*)ex.b_gu, h, ex.act,
      q4_group(ex.fmt), status);
  return cudaGetLastError();
}

cudaError_t launch_down_q4_mma(const void* h, const int32_t* row_off, const int32_t* tile_off,
                               int BM, int R, const moe_experts& ex, void* ys, int* status,
                               cudaStream_t s) {
  const long long tiles = max_tiles(R, ex.E, BM);
  if (tiles <= 0) return cudaSuccess;
  if (tiles > 65535) return cudaErrorInvalidConfiguration;
  dim3 grid(ex.d / 16, (unsigned)tiles);
  launch_pdl(gemv_q4_mma_kernel<false>, grid, kMmaWarps * 32, 0, s, 
      (const __half*)h, nullptr, row_off, tile_off, BM, ex.E, ex.d, ex.F,
      (const uint32_t*)ex.w_dn, (const uint16_t*)ex.s_dn, (const uint16_t*)ex.b_dn, ys,
      MOE_ACT_SWIGLU, q4_group(ex.fmt), status);
  return cudaGetLastError();
}

}  // namespace moe
