// Fused decode layer: the whole forward for a few tokens in one launch.
//
// mlxcel PR #275, "What it does": the decode layer as one single-threadgroup
// kernel (router, top-k, gathered experts, weighted sum) instead of a chain
// of launches; DS4Server issue #112 keeps the weight-streaming kernels for
// T*k/E small. On the B200 one thread block cannot stream the selected
// experts' weights fast enough, so this is one *cooperative* launch of one
// CTA per SM with two grid-wide barriers:
//
//   phase A  router logits x . W_r^T + b (one expert per CTA, one warp per
//            token) and x converted to fp16 (shared by all CTAs)
//   -- grid barrier --
//   phase B  every CTA repeats the top-k of all tokens (warp max of
//            orderable keys, lowest expert index first on ties) and the
//            stable counting sort of the T*k routed rows in shared memory
//            (CTA 0 writes the tables to the workspace); then gate|up + SwiGLU:
//            a work item is 8 features of one active expert (its 8 gate and
//            8 up weight rows), one warp per item, mma.sync m16n8k16 fp16
//            with fp32 accumulation; h goes to global memory in fp16
//   -- grid barrier --
//   phase C  down + combine: a work item is 16 output features; its warps
//            take the active experts in turn, multiply their h rows by the
//            16 weight rows and add w[t][j] * ys into per-warp partial sums
//            in shared memory, which are then added in warp order: no
//            atomics, deterministic
//
// The weight rows of every item are streamed by a producer warp with 1-D bulk
// copies (cp.async.bulk) into a ring of shared-memory slots, so each SM keeps
// up to ~180 KB of weights in flight. The producer knows the item sequence of
// its CTA (it repeats the same computation) and prefetches phase C's weights
// while phase B still runs. Every wait is bounded (~1 s): on expiry the status
// word gets MOE_ERR_TIMEOUT and the kernel returns.
#include <cuda_fp16.h>

#include "common.cuh"
#include "launch.h"

namespace moe {
namespace dec {

constexpr int kCw = 8;                        // compute warps
constexpr int kThreads = (kCw + 1) * 32;      // + the producer warp
constexpr int kMaxT = 32;                     // tokens
constexpr int kMaxR = 256;                    // routed rows T*k
constexpr int kMaxE = 256;                    // experts (top-k keeps E/32 keys per lane)
constexpr int kSlots = 10;                    // weight ring slots (>= kCw)
constexpr int kSlotBytes = 18 * 1024;         // gate|up item: 16 KB of words + 2 KB scales
constexpr long long kWaitCycles = 2000000000LL;

struct Params {
  const __nv_bfloat16* x;                     // [T][d]
  const __nv_bfloat16* wr;                    // [E][d]
  const float* rbias;                         // [E] or null
  const uint32_t* w_gu;                       // [E][2F][d/8] q4 words
  const uint16_t* s_gu;                       // [E][2F][d/64] bf16
  const uint16_t* b_gu;
  const uint32_t* w_dn;                       // [E][d][F/8]
  const uint16_t* s_dn;                       // [E][d][F/64]
  const uint16_t* b_dn;
  int T, d, E, k, F, BM;
  float* logits;                              // [T][E]
  int32_t* topk_idx;                          // [T][k]
  float* topk_w;                              // [T][k]
  uint32_t* order;                            // [R]
  uint32_t* inv_order;                        // [R]
  uint32_t* row_map;                          // [R]
  int32_t* counts;                            // [E]
  int32_t* row_off;                           // [E+1]
  int32_t* tile_off;                          // [E+1]
  __half* x16;                                // [T][d]
  __half* h;                                  // [R][F]
  __nv_bfloat16* y;                           // [T][d]
  unsigned* sync;                             // grid barrier counter, zero before launch
  int* status;
};

// ------------------------------------------------------------------ PTX

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// bounded wait; false when it ran out or (honor_abort) the kernel is aborting
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int* status, bool honor_abort = true) {
  if (mbar_try(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try(bar, parity)) return true;
    if ((i & 15u) == 0) {
      if (honor_abort && *abort_flag) return false;
      if (clock64() - t0 > kWaitCycles) {
        *abort_flag = 1;
        report_status(status, MOE_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// 1-D bulk copy global -> shared, completing on an mbarrier (addresses 16-byte
// aligned, size a multiple of 16)
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

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
// a bf16 value (low 16 bits) as an fp16 pair holding it twice
__device__ __forceinline__ uint32_t h2_from_bf16(uint32_t v16) {
  const float f = __uint_as_float(v16 << 16);
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %1;" : "=r"(d) : "f"(f));
  return d;
}
// 8 nibbles of one word -> fp16 pairs (e0,e1) (e2,e3) (e4,e5) (e6,e7) of
// s*q + b, rounded once: q goes into the mantissa of fp16 1024.0 (exact),
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

// Orderable 32-bit image of a float: larger float -> larger key; -0 -> +0;
// NaN -> 0 (below -inf)
__device__ __forceinline__ uint32_t order_key(float v) {
  if (v == 0.0f) v = 0.0f;
  const uint32_t u = __float_as_uint(v);
  if (isnan(v)) return 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long w = __shfl_xor_sync(0xffffffffu, v, o);
    v = w > v ? w : v;
  }
  return v;
}

// named barrier of the compute warps (the producer warp keeps streaming)
__device__ __forceinline__ void compute_sync() {
  asm volatile("bar.sync 1, %0;" ::"r"(kCw * 32) : "memory");
}

// Grid-wide barrier of the compute warps of all CTAs: a counter that only
// grows (zeroed before the launch); barrier n waits for n * gridDim.x
// arrivals. Bounded: on expiry the status gets MOE_ERR_TIMEOUT.
__device__ __forceinline__ bool grid_barrier(unsigned* ctr, unsigned n, volatile int* abort_flag,
                                             int* status) {
  compute_sync();
  __shared__ int s_ok;
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(ctr, 1u);
    const unsigned target = n * gridDim.x;
    const long long t0 = clock64();
    int ok = 1;
    for (;;) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
      if (v >= target) break;
      if (*abort_flag || clock64() - t0 > kWaitCycles) {
        if (!*abort_flag) report_status(status, MOE_ERR_TIMEOUT);
        *abort_flag = 1;
        ok = 0;
        break;
      }
    }
    __threadfence();
    s_ok = ok;
  }
  compute_sync();
  return s_ok != 0;
}

// One warp, 16 weight rows in shared memory (rows g of group `a` and of
// group `b` for lane (g, c): the m16 A rows g and g + 8), K elements, against
// one group of 8 token rows read from global memory (this lane's row `xrow`,
// zero when !xvalid). mma.sync m16n8k16 fp16, fp32 accumulation into acc:
// acc[0..1] row a for tokens 2c, 2c+1, acc[2..3] row b. Inside the 16-wide
// K slice m of a 128-element step, fragment columns (2c, 2c+1, 2c+8, 2c+9)
// are elements c*32 + 4m + (0..3) for A and B alike, so both come from
// contiguous loads. The token rows were written earlier in this launch (by
// any CTA, before a grid barrier) and are not written again, so plain loads
// may keep them in L1 -- every item of a token reads the same rows -- but
// the read-only path may not; PD steps of them are in flight at once.
template <int PD>
__device__ __forceinline__ void warp_mma_rows16(const uint32_t* wa, const uint32_t* wb,
                                                const uint16_t* sa, const uint16_t* ba,
                                                const uint16_t* sb, const uint16_t* bb,
                                                const __half* xrow, bool xvalid, int K, int c,
                                                float* acc) {
  const int nst = K / 128;
  uint4 xq[PD][4];
  // four independent accumulator chains (K slice m goes to chain m % 4),
  // added at the end: one chain would serialise the 8 MMAs of a step
  float ch[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) ch[i][j] = 0.f;
  auto load = [&](uint4 (&v)[4], int st) {
    const int k0 = st * 128 + c * 32;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      v[i] = xvalid ? *reinterpret_cast<const uint4*>(xrow + k0 + i * 8) : make_uint4(0, 0, 0, 0);
  };
  auto step = [&](const uint4 (&v)[4], int st) {
    const int k0 = st * 128 + c * 32;
    const uint4 wl = *reinterpret_cast<const uint4*>(wa + k0 / 8);
    const uint4 wh = *reinterpret_cast<const uint4*>(wb + k0 / 8);
    const int grp = k0 / 64;
    const uint32_t sl = h2_from_bf16(sa[grp]), bl = h2_from_bf16(ba[grp]);
    const uint32_t sh = h2_from_bf16(sb[grp]), bh = h2_from_bf16(bb[grp]);
    const uint32_t wlw[4] = {wl.x, wl.y, wl.z, wl.w};
    const uint32_t whw[4] = {wh.x, wh.y, wh.z, wh.w};
#pragma unroll
    for (int qw = 0; qw < 4; ++qw) {            // word qw: K slices m = 2qw, 2qw + 1
      uint32_t dl[4], dh[4];
      q4_word_f16(wlw[qw], sl, bl, dl);
      q4_word_f16(whw[qw], sh, bh, dh);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const uint32_t av[4] = {dl[2 * half], dh[2 * half], dl[2 * half + 1], dh[2 * half + 1]};
        const uint4 x = v[qw];                  // slice m = 2qw + half: words 2m, 2m + 1
        mma_16816(ch[(2 * qw + half) & 3], av, half ? x.z : x.x, half ? x.w : x.y);
      }
    }
  };
#pragma unroll
  for (int i = 0; i < PD; ++i)
    if (i < nst) load(xq[i], i);
  for (int st0 = 0; st0 < nst; st0 += PD) {
#pragma unroll
    for (int i = 0; i < PD; ++i) {
      const int st = st0 + i;
      if (st < nst) {
        step(xq[i], st);
        if (st + PD < nst) load(xq[i], st + PD);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) acc[j] += (ch[0][j] + ch[1][j]) + (ch[2][j] + ch[3][j]);
}

// Top-k of tokens warp, warp + kCw, ... (at most TPW per warp, all at once)
// from the logits in global memory; results into shared memory.
template <int VPL, int TPW>
__device__ __forceinline__ void topk_tokens(const Params& p, int warp, int lane, int* s_idx,
                                            float* s_w) {
  const int E = p.E, k = p.k;
  unsigned long long key[TPW][VPL];
  int my_e[TPW];
#pragma unroll
  for (int q = 0; q < TPW; ++q) {
    const int t = warp + q * kCw;
    const float* row = p.logits + (size_t)(t < p.T ? t : 0) * E;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = lane + 32 * i;
      key[q][i] = (t < p.T && e < E) ? (((unsigned long long)order_key(__ldcg(row + e)) << 32) |
                                        (0xFFFFFFFFu - (uint32_t)e))
                                     : 0ull;
    }
    my_e[q] = -1;
  }
  for (int j = 0; j < k; ++j) {
#pragma unroll
    for (int q = 0; q < TPW; ++q) {
      unsigned long long best = 0ull;
#pragma unroll
      for (int i = 0; i < VPL; ++i) best = key[q][i] > best ? key[q][i] : best;
      best = warp_max_u64(best);
      const int e = (int)(0xFFFFFFFFu - (uint32_t)(best & 0xFFFFFFFFull));
      if (lane == j) my_e[q] = e;
#pragma unroll
      for (int i = 0; i < VPL; ++i)
        if (lane + 32 * i == e) key[q][i] = 0ull;
    }
  }
#pragma unroll
  for (int q = 0; q < TPW; ++q) {
    const int t = warp + q * kCw;
    if (t >= p.T) continue;
    const float* row = p.logits + (size_t)t * E;
    const float m = __ldcg(row + __shfl_sync(0xffffffffu, my_e[q], 0));
    const float ex = lane < k ? __expf(__ldcg(row + my_e[q]) - m) : 0.f;
    const float den = warp_sum(ex);
    if (lane < k) {
      s_idx[t * k + lane] = my_e[q];
      s_w[t * k + lane] = ex / den;
    }
  }
}

// ------------------------------------------------------------------ kernel

// Work items of this CTA, identical in every role: gate|up items gi = c,
// c + G, ... < nA * F/8 (active expert gi / (F/8), features 8 * (gi % (F/8))),
// then for each down item ob = c, c + G, ... < d/16 one sub-item per active
// expert. The ring sequence number s counts them in that order.
struct Plan {
  int nA;       // active experts
  int nB;       // gate|up items of this CTA
  int nC;       // down items of this CTA
  int fpb;      // feature blocks per expert (F / 8)
};

__device__ __forceinline__ Plan make_plan(const Params& p, int nA) {
  Plan pl;
  pl.nA = nA;
  pl.fpb = p.F / 8;
  const int G = gridDim.x, c = blockIdx.x;
  const int totB = nA * pl.fpb, totC = p.d / 16;
  pl.nB = c < totB ? (totB - c + G - 1) / G : 0;
  pl.nC = c < totC ? (totC - c + G - 1) / G : 0;
  return pl;
}

__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                             ~(uintptr_t)127);
  __shared__ uint64_t full[kSlots], empty[kSlots];
  __shared__ int s_idx[kMaxR];          // expert of routed row t*k + j
  __shared__ float s_w[kMaxR];          // its weight
  __shared__ int s_roff[kMaxE + 1];     // rows of expert e: s_roff[e] .. s_roff[e+1]-1
  __shared__ int s_rows[kMaxR];         // sorted row r -> routed row t*k + j
  __shared__ int s_act[kMaxE];          // active experts, increasing
  __shared__ int s_nact;
  __shared__ float s_y[kCw][kMaxT][16]; // down: per-warp partial sums
  __shared__ volatile int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.T, d = p.d, E = p.E, k = p.k, F = p.F;
  const int R = T * k;
  const int G = gridDim.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(smem_u32(full + i), 1);
      mbar_init(smem_u32(empty + i), 1);
    }
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  pdl_wait();
  pdl_launch();
  __syncthreads();

  // ---------------------------------------------------------------- phase A
  // x -> fp16 (8 values per thread, all CTAs share the rows)
  {
    const int n8 = T * d / 8;
    const uint4* xs = reinterpret_cast<const uint4*>(p.x);
    uint4* xo = reinterpret_cast<uint4*>(p.x16);
    for (int i = blockIdx.x * kThreads + threadIdx.x; i < n8; i += G * kThreads) {
      const uint4 v = xs[i];
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float a = __uint_as_float(w4[j] << 16), b = __uint_as_float(w4[j] & 0xFFFF0000u);
        if (!(fabsf(a) < 65520.f && fabsf(b) < 65520.f)) report_status(p.status, MOE_ERR_RANGE);
        asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(o[j]) : "f"(b), "f"(a));
      }
      xo[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  // router logits: expert e of this CTA, token t per compute warp, fp32 sums
  // of exact bf16 products
  if (warp < kCw) {
    for (int e = blockIdx.x; e < E; e += G) {
      const uint4* wrow = reinterpret_cast<const uint4*>(p.wr + (size_t)e * d);
      for (int t = warp; t < T; t += kCw) {
        const uint4* xrow = reinterpret_cast<const uint4*>(p.x + (size_t)t * d);
        float acc = 0.f;
        for (int c8 = lane; c8 < d / 8; c8 += 32) {
          const uint4 a = __ldg(wrow + c8), b = xrow[c8];
          const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 fa = bf16x2_to_f32x2(wa[j]), fb = bf16x2_to_f32x2(wb[j]);
            acc = fmaf(fa.x, fb.x, acc);
            acc = fmaf(fa.y, fb.y, acc);
          }
        }
        acc = warp_sum(acc);
        if (lane == 0) p.logits[(size_t)t * E + e] = acc + (p.rbias ? p.rbias[e] : 0.f);
      }
    }
  }
  __syncthreads();
  bool ok = true;
  if (warp < kCw) ok = grid_barrier(p.sync, 1, &s_abort, p.status);
  __syncthreads();
  if (s_abort) ok = false;

  // ---------------------------------------------------------------- routing
  // top-k of every token (all CTAs alike): lane l keeps keys of experts
  // l, l + 32, ...; k rounds of a warp max pick the best remaining expert,
  // the lowest index among equal logits; weights exp(L - Lmax) / sum. A warp
  // takes tokens w, w + 8, w + 16, w + 24 together (independent chains).
  if (ok && warp < kCw) {
    if (T <= kCw) {
      if (E <= 128) topk_tokens<4, 1>(p, warp, lane, s_idx, s_w);
      else topk_tokens<kMaxE / 32, 1>(p, warp, lane, s_idx, s_w);
    } else {
      if (E <= 128) topk_tokens<4, kMaxT / kCw>(p, warp, lane, s_idx, s_w);
      else topk_tokens<kMaxE / 32, kMaxT / kCw>(p, warp, lane, s_idx, s_w);
    }
  }
  __syncthreads();
  // stable counting sort of the routed rows by expert (all CTAs alike), by
  // warp 0: chunks of 32 rows in order; __match_any_sync groups the lanes of
  // one expert, a row's rank within its expert is the count carried from
  // earlier chunks plus the lanes of its group below it
  if (ok && warp == 0) {
    for (int e = lane; e < E; e += 32) s_roff[e] = 0;     // per-expert counts for now
    __syncwarp();
    for (int c0 = 0; c0 < R; c0 += 32) {
      const int i = c0 + lane;
      const int e = i < R ? s_idx[i] : -1 - lane;
      const unsigned grp = __match_any_sync(0xffffffffu, e);
      const int below = __popc(grp & ((1u << lane) - 1u));
      const int base = i < R ? s_roff[e] : 0;
      __syncwarp();
      if (i < R) {
        s_rows[i] = base + below;                          // rank within expert, for now
        if (below == 0) s_roff[e] = base + __popc(grp);
      }
      __syncwarp();
    }
    // exclusive scan of the counts (lane l owns experts 8l .. 8l + 7) and
    // the list of experts with rows, in increasing order
    constexpr int PER = kMaxE / 32;
    int cnt[PER], tot = 0, act = 0;
#pragma unroll
    for (int q = 0; q < PER; ++q) {
      const int e = lane * PER + q;
      cnt[q] = e < E ? s_roff[e] : 0;
      tot += cnt[q];
      act += cnt[q] > 0;
    }
    int itot = tot, iact = act;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a1 = __shfl_up_sync(0xffffffffu, itot, o), a2 = __shfl_up_sync(0xffffffffu, iact, o);
      if (lane >= o) { itot += a1; iact += a2; }
    }
    int off = itot - tot, apos = iact - act;
    __syncwarp();
#pragma unroll
    for (int q = 0; q < PER; ++q) {
      const int e = lane * PER + q;
      if (e < E) {
        s_roff[e] = off;
        if (cnt[q] > 0) s_act[apos++] = e;
      }
      off += cnt[q];
    }
    if (lane == 31) {
      s_roff[E] = off;
      s_nact = apos;
    }
  }
  __syncthreads();
  if (ok) {
    int rk[(kMaxR + kThreads - 1) / kThreads];
#pragma unroll
    for (int q = 0; q * kThreads < kMaxR; ++q) {
      const int i = q * kThreads + threadIdx.x;
      rk[q] = i < R ? s_roff[s_idx[i]] + s_rows[i] : 0;
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q * kThreads < kMaxR; ++q) {
      const int i = q * kThreads + threadIdx.x;
      if (i < R) s_rows[rk[q]] = i;                         // sorted row -> routed row
    }
  }
  __syncthreads();
  // the workspace tables, as moe_route and moe_sort_rows write them
  if (ok && blockIdx.x == 0) {
    for (int i = threadIdx.x; i < R; i += kThreads) {
      p.topk_idx[i] = s_idx[i];
      p.topk_w[i] = s_w[i];
      const uint32_t slot = (uint32_t)s_rows[i];
      p.order[i] = slot;
      p.inv_order[slot] = (uint32_t)i;
      p.row_map[i] = slot / (uint32_t)k;
    }
    for (int e = threadIdx.x; e <= E; e += kThreads) {
      p.row_off[e] = s_roff[e];
      if (e < E) p.counts[e] = s_roff[e + 1] - s_roff[e];
    }
    if (warp == 0) {          // tile offsets: a warp scan of ceil(count / BM)
      int carry = 0;
      for (int e0 = 0; e0 <= E; e0 += 32) {
        const int e = e0 + lane;
        const int n = e < E ? (s_roff[e + 1] - s_roff[e] + p.BM - 1) / p.BM : 0;
        int incl = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int a1 = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += a1;
        }
        if (e <= E) p.tile_off[e] = carry + incl - n;
        carry += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
  }
  __syncthreads();
  const Plan pl = make_plan(p, s_nact);
  const int nseq = pl.nB + pl.nC * pl.nA;      // ring sequence of this CTA

  if (warp == kCw) {
    // ------------------------------------------------------------ producer
    // one thread streams every item's weight rows (and their scales and
    // biases) into ring slot s % kSlots, after the item kSlots earlier in the
    // sequence has released it
    if (lane == 0 && ok) {
      int s = 0;
      for (; s < nseq; ++s) {
        const int slot = s % kSlots;
        if (s >= kSlots &&
            !mbar_wait(smem_u32(empty + slot), ((s / kSlots) - 1) & 1, &s_abort, p.status))
          break;
        const uint32_t dst = smem_u32(ring + slot * kSlotBytes);
        const uint32_t bar = smem_u32(full + slot);
        if (s < pl.nB) {
          const int gi = blockIdx.x + s * G;
          const int e = s_act[gi / pl.fpb], f0 = (gi % pl.fpb) * 8;
          const size_t rg = (size_t)e * 2 * F + f0, ru = rg + F;   // first gate / up row
          const uint32_t wb = 8u * (uint32_t)(d / 2), sb = 8u * (uint32_t)(d / 32);
          mbar_expect_tx(bar, 2 * wb + 4 * sb);
          bulk_g2s(dst, p.w_gu + rg * (d / 8), wb, bar);
          bulk_g2s(dst + wb, p.w_gu + ru * (d / 8), wb, bar);
          bulk_g2s(dst + 2 * wb, p.s_gu + rg * (d / 64), sb, bar);
          bulk_g2s(dst + 2 * wb + sb, p.s_gu + ru * (d / 64), sb, bar);
          bulk_g2s(dst + 2 * wb + 2 * sb, p.b_gu + rg * (d / 64), sb, bar);
          bulk_g2s(dst + 2 * wb + 3 * sb, p.b_gu + ru * (d / 64), sb, bar);
        } else {
          const int sc = s - pl.nB;
          const int m = sc / pl.nA, a = sc - m * pl.nA;
          const int ob = blockIdx.x + m * G;
          const size_t r = (size_t)s_act[a] * d + (size_t)ob * 16;     // first of 16 rows
          const uint32_t wb = 16u * (uint32_t)(F / 2), sb = 16u * (uint32_t)(F / 32);
          mbar_expect_tx(bar, wb + 2 * sb);
          bulk_g2s(dst, p.w_dn + r * (F / 8), wb, bar);
          bulk_g2s(dst + wb, p.s_dn + r * (F / 64), sb, bar);
          bulk_g2s(dst + wb + sb, p.b_dn + r * (F / 64), sb, bar);
        }
      }
      // copies in flight land before the CTA may exit (bounded, also when
      // aborting)
      for (int i = 0; i < kSlots && i < s; ++i) {
        const int last = s - 1 - i;
        mbar_wait(smem_u32(full + last % kSlots), (last / kSlots) & 1, &s_abort, p.status, false);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ compute warps
    const int g = lane >> 2, c = lane & 3;
    // gate|up + SwiGLU: item s of this CTA, one warp per item. Lane (g, c)
    // holds gate row g and up row g of the 8 features (the m16 A rows g and
    // g + 8) and token g of each group of 8 (B columns); inside the 16-wide
    // K slice m of a 128-element step, fragment columns (2c, 2c+1, 2c+8,
    // 2c+9) are elements c*32 + 4m + (0..3) for A and B alike, so both come
    // from contiguous loads.
    for (int s = warp; s < pl.nB && ok; s += kCw) {
      const int slot = s % kSlots;
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(full + slot), (s / kSlots) & 1, &s_abort,
                                              p.status));
      if (!ok) break;
      const uint8_t* sp = ring + slot * kSlotBytes;
      const int gi = blockIdx.x + s * G;
      const int f0 = (gi % pl.fpb) * 8;
      const int e = s_act[gi / pl.fpb];
      const int r0 = s_roff[e], nv = s_roff[e + 1] - r0;
      const uint32_t* wg = reinterpret_cast<const uint32_t*>(sp) + g * (d / 8);
      const uint32_t* wu = reinterpret_cast<const uint32_t*>(sp + 4 * d) + g * (d / 8);
      const uint16_t* sg = reinterpret_cast<const uint16_t*>(sp + 8 * d) + g * (d / 64);
      const uint16_t* su = sg + 8 * (d / 64);
      const uint16_t* bg = su + 8 * (d / 64);
      const uint16_t* bu = bg + 8 * (d / 64);
      // 8 token rows per pass; the weights stay in shared memory
      for (int q = 0; q * 8 < nv; ++q) {
        const int n = q * 8 + g;
        const bool xv = n < nv;
        const __half* xr = p.x16 + (size_t)(xv ? s_rows[r0 + n] / k : 0) * d;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        warp_mma_rows16<4>(wg, wu, sg, bg, su, bu, xr, xv, d, c, acc);
        // lane (g, c): gate (acc[0..1]) and up (acc[2..3]) of feature f0 + g
        // for the expert's tokens q*8 + 2c, q*8 + 2c + 1
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int n2 = q * 8 + 2 * c + j;
          if (n2 < nv) {
            const float v = swiglu(acc[j], acc[2 + j]);
            if (!(fabsf(v) < 65520.f)) report_status(p.status, MOE_ERR_RANGE);
            p.h[(size_t)(r0 + n2) * F + f0 + g] = __float2half_rn(v);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(empty + slot));
    }
    // all of h is written before any CTA reads it
    if (!grid_barrier(p.sync, 2, &s_abort, p.status)) ok = false;

    // down + combine: item ob (16 output features); warp w takes active
    // experts w, w + 8, ...: rows o0 + g and o0 + 8 + g (A rows g, g + 8)
    // against the expert's h rows (B columns), then y[t][o] += w[t][j] * ys
    // into this warp's partial sums
    // (every compute warp runs every iteration: the named barriers inside
    // need all of them, so a failed wait only skips the work)
    for (int m = 0; m < pl.nC; ++m) {
      const int ob = blockIdx.x + m * G;
      for (int i = threadIdx.x; i < kCw * kMaxT * 16; i += kCw * 32) (&s_y[0][0][0])[i] = 0.f;
      compute_sync();
      for (int a = warp; a < pl.nA && ok; a += kCw) {
        const int s = pl.nB + m * pl.nA + a;
        const int slot = s % kSlots;
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(full + slot), (s / kSlots) & 1, &s_abort,
                                                p.status));
        if (!ok) break;
        const uint8_t* sp = ring + slot * kSlotBytes;
        const int e = s_act[a];
        const int r0 = s_roff[e], nv = s_roff[e + 1] - r0;
        const uint32_t* wl_ = reinterpret_cast<const uint32_t*>(sp) + g * (F / 8);
        const uint32_t* wh_ = reinterpret_cast<const uint32_t*>(sp) + (g + 8) * (F / 8);
        const uint16_t* sc_ = reinterpret_cast<const uint16_t*>(sp + 8 * F);
        const uint16_t* bi_ = sc_ + 16 * (F / 64);
        for (int q = 0; q * 8 < nv; ++q) {
          const int n = q * 8 + g;
          const bool hvld = n < nv;
          const __half* hr = p.h + (size_t)(hvld ? r0 + n : 0) * F;
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
          warp_mma_rows16<4>(wl_, wh_, sc_ + g * (F / 64), bi_ + g * (F / 64),
                             sc_ + (g + 8) * (F / 64), bi_ + (g + 8) * (F / 64), hr, hvld, F, c,
                             acc);
          // lane (g, c): rows o0 + g (acc[0..1]) and o0 + 8 + g (acc[2..3])
          // for the expert's tokens q*8 + 2c, q*8 + 2c + 1
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int n2 = q * 8 + 2 * c + j;
            if (n2 < nv) {
              const int i = s_rows[r0 + n2];
              const int t = i / k;
              const float wt = s_w[i];
              s_y[warp][t][g] += wt * acc[j];
              s_y[warp][t][g + 8] += wt * acc[2 + j];
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(empty + slot));
      }
      compute_sync();
      if (s_abort) ok = false;
      for (int i = threadIdx.x; i < T * 16 && !s_abort; i += kCw * 32) {
        const int t = i >> 4, o = i & 15;
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kCw; ++w) v += s_y[w][t][o];
        p.y[(size_t)t * d + ob * 16 + o] = __float2bfloat16_rn(v);
      }
      compute_sync();
    }
  }
}

// ------------------------------------------------------------------ host

static int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

}  // namespace dec

bool decode_fused_ok(int T, int k, int E, int d, int F, int fmt, int dt) {
  using namespace dec;
  return fmt == MOE_W_Q4G64 && dt == MOE_BF16 && T >= 1 && T <= kMaxT && T * k <= kMaxR &&
         E <= kMaxE && k <= 32 && d % 128 == 0 && F % 128 == 0 && d <= 2048 && F <= 2048;
}

size_t decode_smem_bytes() { return dec::kSlots * dec::kSlotBytes + 128; }

cudaError_t launch_decode_fused(const void* x, const void* w_router, const float* bias,
                                const moe_experts& ex, int T, int k, int BM, float* logits,
                                int32_t* idx, float* w, uint32_t* order, uint32_t* inv_order,
                                uint32_t* row_map, int32_t* counts, int32_t* row_off,
                                int32_t* tile_off, void* x16, void* h, void* y, unsigned* sync,
                                int* status, cudaStream_t s) {
  using namespace dec;
  if (!decode_fused_ok(T, k, ex.E, ex.d, ex.F, ex.fmt, MOE_BF16)) return cudaErrorNotSupported;
  const int G = sm_count();
  if (G <= 0) return cudaErrorNoDevice;
  Params p{};
  p.x = (const __nv_bfloat16*)x;
  p.wr = (const __nv_bfloat16*)w_router;
  p.rbias = bias;
  p.w_gu = (const uint32_t*)ex.w_gu;
  p.s_gu = (const uint16_t*)ex.s_gu;
  p.b_gu = (const uint16_t*)ex.b_gu;
  p.w_dn = (const uint32_t*)ex.w_dn;
  p.s_dn = (const uint16_t*)ex.s_dn;
  p.b_dn = (const uint16_t*)ex.b_dn;
  p.T = T;
  p.d = ex.d;
  p.E = ex.E;
  p.k = k;
  p.F = ex.F;
  p.BM = BM;
  p.logits = logits;
  p.topk_idx = idx;
  p.topk_w = w;
  p.order = order;
  p.inv_order = inv_order;
  p.row_map = row_map;
  p.counts = counts;
  p.row_off = row_off;
  p.tile_off = tile_off;
  p.x16 = (__half*)x16;
  p.h = (__half*)h;
  p.y = (__nv_bfloat16*)y;
  p.sync = sync;
  p.status = status;
  const size_t smem = decode_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  // the barrier counter starts from zero every launch
  if ((e = cudaMemsetAsync(sync, 0, sizeof(unsigned), s)) != cudaSuccess) return e;
  // one CTA per SM, all resident at once (cooperative launch), after the
  // previous kernel on the stream (programmatic overlap of the prologue)
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)G);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_kernel, p);
}

}  // namespace moe
