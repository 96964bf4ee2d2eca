// Fused decode layer: the whole forward for a few tokens in one launch.
//
// mlxcel PR #275, "What it does": the decode layer as one single-threadgroup
// kernel (router, top-k, gathered experts, weighted sum) instead of a chain
// of launches; DS4Server issue #112 keeps the weight-streaming kernels for
// T*k/E small. On the B200 one thread block cannot stream the selected
// experts' weights fast enough, so this is one *cooperative* launch of one
// CTA per SM with three grid-wide barriers:
//
//   phase A  router logits x . W_r^T + b (a warp per expert and token) and x
//            converted to fp16 (shared by all CTAs)
//   -- grid barrier --
//   phase B  every CTA repeats the top-k of all tokens (one warp per token,
//            two warp reductions per selected expert, lowest expert index
//            first on ties) and the stable counting sort of the T*k routed
//            rows in shared memory; then gate|up + SwiGLU: a work item is 8
//            features of one active expert (its 8 gate and 8 up weight rows)
//   -- grid barrier --
//   phase C  down: a work item is 16 output features of one active expert,
//            written to ys (fp16, sorted row order)
//   -- grid barrier --
//   phase D  combine: y[t] = sum over j of w[t][j] * ys[inv_order[t*k + j]]
//            in j order, one thread per 8 outputs: no atomics, deterministic
//
// Each CTA takes a contiguous range of the gate|up items and of the down
// items (expert-major), so consecutive items share an expert and its token or
// h rows stay in L1. The compute warps form groups of four. A group takes one
// work item at a time and splits its K range: warp i of the group multiplies
// the 128-wide K steps i, i + 4, ... (mma.sync m16n8k16, fp16 operands, fp32
// accumulation), so an item's latency is a quarter of one warp's, and every
// warp of the SM has work even when the SM has only a few items. The four
// partial accumulators are added in group order through shared memory.
//
// The weight rows of every item are streamed by a producer warp with 1-D bulk
// copies (cp.async.bulk) into a ring of shared-memory slots, so each SM keeps
// up to ~180 KB of weights in flight. The producer knows the item sequence of
// its CTA (it repeats the same computation) and prefetches phase C's weights
// while phase B still runs. Every wait is bounded (~1 s): on expiry the status
// word gets MOE_ERR_TIMEOUT and the kernel returns.
//
// The fp16 token rows (x16) and h are stored with every 8 consecutive elements
// in the order (0,4,1,5,2,6,3,7): the K order in which the dequantisation
// produces weight pairs. ys, y and the tables have their plain layouts.
#include <cuda_fp16.h>

#include "common.cuh"
#include "launch.h"

namespace moe {
namespace dec {

constexpr int kCw = 16;                       // compute warps
constexpr int kGw = 4;                        // warps per group (K split)
constexpr int kNg = kCw / kGw;                // groups
constexpr int kThreads = (kCw + 1) * 32;      // + the producer warp
constexpr int kMaxT = 32;                     // tokens
constexpr int kMaxR = 256;                    // routed rows T*k
constexpr int kMaxE = 256;                    // experts (top-k keeps E/32 logits per lane)
constexpr int kSlots = 10;                    // weight ring slots
// gate|up item at d = 2048: 16 KB of words + up to 4 KB of scales and biases
// (group 32)
constexpr int kSlotBytes = 20 * 1024;
constexpr long long kWaitCycles = 2000000000LL;

// shared memory after the ring: the groups' partial accumulators (double
// buffered per group)
constexpr int kRedBytes = 2 * kNg * kGw * 32 * 4 * 4;

struct Params {
  const uint16_t* x;                          // [T][d] bf16, or fp16 when xf16
  const uint16_t* wr;                         // [E][d] same type as x
  const float* rbias;                         // [E] or null
  const uint32_t* w_gu;                       // [E][2F][d/8] q4 words
  const uint16_t* s_gu;                       // [E][2F][d/gs] bf16
  const uint16_t* b_gu;
  const uint32_t* w_dn;                       // [E][d][F/8]
  const uint16_t* s_dn;                       // [E][d][F/gs]
  const uint16_t* b_dn;
  int T, d, E, k, F, BM;
  int act;                                    // the GLU's gate activation (moe_act)
  int gs, gshift;                             // elements per q4 scale (32, 64, 128), log2
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
  __half* ys;                                 // [R][d], sorted row order
  uint16_t* y;                                // [T][d] same type as x
  int xf16;                                   // activations are fp16 (else bf16)
  unsigned* sync;                             // grid barrier counter, zero before launch
  int* status;
  long long wait_limit;                       // SM cycles a wait for work may take
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
// bounded wait (at most `limit` SM cycles); false when it ran out or
// (honor_abort) the kernel is aborting. Waits for work take the launch's bound
// (Params::wait_limit); the producer's final wait for its copies in flight
// keeps the full bound, so no copy lands after the CTA has exited.
__device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                       int* status, bool honor_abort = true,
                                       long long limit = kWaitCycles) {
  if (mbar_try(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try(bar, parity)) return true;
    if ((i & 15u) == 0) {
      if (honor_abort && *abort_flag) return false;
      if (clock64() - t0 > limit) {
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
// 8 nibbles of one word -> fp16 pairs (e0,e4) (e1,e5) (e2,e6) (e3,e7) of
// s*q + b, rounded once. Nibbles 0 and 4 (bits 0-3, 16-19) are ORed into the
// mantissa of fp16 1024.0, whose last place is 1; nibbles 1 and 5 (bits 4-7,
// 20-23) into that of fp16 64.0, whose last place is 1/16, so both pairs
// read magic + q. A byte permute puts bytes 1 and 3 (e3:e2, e7:e6) under the
// exponent of 1024, giving 1024 + 16 e3 + e2; its bits 4-7 ORed into 64.0
// give 64 + e3, and e2 = (1024 + 16 e3 + e2) - 16 (64 + e3) exactly. The
// magic is subtracted exactly and one fused multiply-add applies scale and
// bias: 4 integer and 8 fp16 operations per 8 weights.
__device__ __forceinline__ void q4_word_perm(uint32_t w, uint32_t s2, uint32_t b2, uint32_t* o) {
  const uint32_t c1024 = 0x64006400u, c64 = 0x54005400u, m16 = 0xCC00CC00u;   // -16.0
  const uint32_t hi = __byte_perm(w, 0x64646464u, 0x4341);
  const uint32_t d = (hi & 0x00F000F0u) | c64;
  o[0] = h2_fma(h2_sub((w & 0x000F000Fu) | c1024, c1024), s2, b2);
  o[1] = h2_fma(h2_sub((w & 0x00F000F0u) | c64, c64), s2, b2);
  o[2] = h2_fma(h2_fma(d, m16, hi), s2, b2);
  o[3] = h2_fma(h2_sub(d, c64), s2, b2);
}

// Orderable 32-bit image of a float: larger float -> larger key; -0 -> +0;
// NaN -> 0 (below -inf, whose key is 0x007FFFFF)
__device__ __forceinline__ uint32_t order_key(float v) {
  if (v == 0.0f) v = 0.0f;
  const uint32_t u = __float_as_uint(v);
  if (isnan(v)) return 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// named barrier of the compute warps (the producer warp keeps streaming)
__device__ __forceinline__ void compute_sync() {
  asm volatile("bar.sync 1, %0;" ::"r"(kCw * 32) : "memory");
}
// named barrier of one group's four warps, returning whether `ok` holds in
// all of them (so a group leaves a loop together)
__device__ __forceinline__ bool group_sync_and(int grp, bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)ok), "r"(2 + grp), "r"(kGw * 32)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void group_sync(int grp) {
  asm volatile("bar.sync %0, %1;" ::"r"(2 + grp), "r"(kGw * 32) : "memory");
}

// Grid-wide barrier of the compute warps of all CTAs: a counter that only
// grows (zeroed before the launch); barrier n waits for n * gridDim.x
// arrivals. Bounded (`limit` SM cycles): on expiry the status gets
// MOE_ERR_TIMEOUT. A CTA that is aborting still arrives, so the others are
// not kept waiting for it.
__device__ __noinline__ bool grid_barrier(unsigned* ctr, unsigned n, volatile int* abort_flag,
                                          int* status, long long limit) {
  compute_sync();
  __shared__ int s_ok;
  if (threadIdx.x == 0) {
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
    asm volatile("red.relaxed.gpu.global.add.u32 [%0], 1;" ::"l"(ctr) : "memory");
    const unsigned target = n * gridDim.x;
    const long long t0 = clock64();
    int ok = 1;
    for (;;) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
      if (v >= target) break;
      if (*abort_flag || clock64() - t0 > limit) {
        if (!*abort_flag) report_status(status, MOE_ERR_TIMEOUT);
        *abort_flag = 1;
        ok = 0;
        break;
      }
    }
    s_ok = ok;
  }
  compute_sync();
  return s_ok != 0;
}

// One warp, 16 weight rows in shared memory (row g of matrix `a` and of
// matrix `b` for lane (g, c): the m16 A rows g and g + 8), against one group
// of 8 token rows read from global memory (this lane's row `xrow`, zero when
// !xvalid), over the 128-wide K steps st0, st0 + sstride, ... < nst. mma.sync
// m16n8k16 fp16, fp32 accumulation into acc: acc[0..1] row a for tokens 2c,
// 2c+1, acc[2..3] row b.
//
// K order: lane c takes elements 32c .. 32c + 31 of a step, four q4 words
// per row, which share one scale and bias (groups of 32, 64 or 128 elements,
// 1 << gshift). Word j gives
// the fp16 pairs (e0,e4) (e1,e5) (e2,e6) (e3,e7); K slice 2j of the step
// takes the first two as fragment columns (2c, 2c+1) and (2c+8, 2c+9), slice
// 2j + 1 the last two. The token rows are stored with every 8 consecutive
// elements in the order (0,4,1,5,2,6,3,7), so one 16-byte load holds the
// matching B fragments of one word. The token rows were written earlier in
// this launch (by any CTA, before a grid barrier) and are not written again,
// so plain loads may keep them in L1 -- the items of an expert read the same
// rows -- but the read-only path may not. Two steps of them are in flight.
__device__ __forceinline__ void warp_mma_steps(const uint8_t* wa, const uint8_t* wb,
                                               const uint16_t* sa, const uint16_t* ba,
                                               const uint16_t* sb, const uint16_t* bb,
                                               const __half* xrow, bool xvalid, int st0, int nst,
                                               int sstride, int gshift, int c, float* acc) {
  float ch[2][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) ch[i][j] = 0.f;
  uint4 xq[2][4];
  auto load = [&](uint4 (&v)[4], int st) {
    const uint4* src = reinterpret_cast<const uint4*>(xrow + st * 128 + c * 32);
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = xvalid ? src[i] : make_uint4(0, 0, 0, 0);
  };
  auto step = [&](const uint4 (&v)[4], int st) {
    const uint4 wl = *reinterpret_cast<const uint4*>(wa + st * 64 + c * 16);
    const uint4 wh = *reinterpret_cast<const uint4*>(wb + st * 64 + c * 16);
    const int grp = (st * 128 + c * 32) >> gshift;
    // scales and biases of rows a and b as fp16 pairs (value, value)
    uint32_t s2, b2;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;"
        : "=r"(s2)
        : "f"(__uint_as_float((uint32_t)sb[grp] << 16)),
          "f"(__uint_as_float((uint32_t)sa[grp] << 16)));
    asm("cvt.rn.f16x2.f32 %0, %1, %2;"
        : "=r"(b2)
        : "f"(__uint_as_float((uint32_t)bb[grp] << 16)),
          "f"(__uint_as_float((uint32_t)ba[grp] << 16)));
    const uint32_t sl = __byte_perm(s2, 0, 0x1010), sh = __byte_perm(s2, 0, 0x3232);
    const uint32_t bl = __byte_perm(b2, 0, 0x1010), bh = __byte_perm(b2, 0, 0x3232);
    const uint32_t wlw[4] = {wl.x, wl.y, wl.z, wl.w}, whw[4] = {wh.x, wh.y, wh.z, wh.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t dl[4], dh[4];
      q4_word_perm(wlw[j], sl, bl, dl);
      q4_word_perm(whw[j], sh, bh, dh);
      const uint32_t a0[4] = {dl[0], dh[0], dl[1], dh[1]};
      const uint32_t a1[4] = {dl[2], dh[2], dl[3], dh[3]};
      mma_16816(ch[0], a0, v[j].x, v[j].y);
      mma_16816(ch[1], a1, v[j].z, v[j].w);
    }
  };
  int st = st0;
  if (st < nst) load(xq[0], st);
  if (st + sstride < nst) load(xq[1], st + sstride);
#pragma unroll 1
  for (; st < nst; st += 2 * sstride) {
    step(xq[0], st);
    if (st + 2 * sstride < nst) load(xq[0], st + 2 * sstride);
    if (st + sstride < nst) {
      step(xq[1], st + sstride);
      if (st + 3 * sstride < nst) load(xq[1], st + 3 * sstride);
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) acc[j] = ch[0][j] + ch[1][j];
}

// Top-k of one token by one warp, from its logits row in global memory;
// results into shared memory. Lane l holds the logits of experts l, l + 32,
// ...; each of the k rounds takes the lane's best remaining expert (largest
// key, the lowest index among equal keys), the warp maximum of those keys,
// and the lowest expert index among the lanes that hold it. The weights are
// exp(L_j - L_max) / sum over the selected, in the lane order of a warp sum.
__device__ __noinline__ void topk_token(const float* row, int E, int k, int lane, int* idx_out,
                                        float* w_out) {
  constexpr int VPL = kMaxE / 32;
  uint32_t key[VPL];
  float val[VPL];
  uint32_t avail = 0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane + 32 * i;
    val[i] = e < E ? __ldcg(row + e) : 0.f;
    key[i] = order_key(val[i]);
    if (e < E) avail |= 1u << i;
  }
  int my_e = 0;
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
  const float m = __shfl_sync(0xffffffffu, my_v, 0);
  const float ex = lane < k ? __expf(my_v - m) : 0.f;
  const float den = warp_sum(ex);
  if (lane < k) {
    idx_out[lane] = my_e;
    w_out[lane] = ex / den;
  }
}

// ------------------------------------------------------------------ kernel

// Work items of this CTA, identical in every role. Gate|up items are numbered
// gi = a * (F/8) + fb over the active experts a (features 8 fb .. 8 fb + 7);
// down items di = a * (d/16) + ob (output features 16 ob .. 16 ob + 15). Each
// CTA takes a contiguous range of each list, so consecutive items share an
// expert and its token (or h) rows stay in L1. The ring sequence number s
// counts the CTA's gate|up items, then its down items; item s is taken by
// compute group s % kNg.
struct Plan {
  int nA;       // active experts
  int fpb;      // feature blocks per expert (F / 8)
  int dr;       // output rows per down item (16 or 32)
  int opb;      // output blocks per expert (d / dr)
  int b0, nB;   // first gate|up item and count
  int c0, nC;   // first down item and count
};

__device__ __forceinline__ Plan make_plan(int d, int F, int gshift, int nA) {
  Plan pl;
  pl.nA = nA;
  pl.fpb = F / 8;
  // 32 rows when they fit a ring slot (their F / 2 bytes of words and 2 F / gs
  // of scales and biases each), so the four warps of a group split an item
  // evenly
  pl.dr = 32 * (F / 2 + 4 * (F >> gshift)) <= kSlotBytes ? 32 : 16;
  pl.opb = d / pl.dr;
  const long long G = gridDim.x, c = blockIdx.x;
  const long long totB = (long long)nA * pl.fpb, totC = (long long)nA * pl.opb;
  pl.b0 = (int)(c * totB / G);
  pl.nB = (int)((c + 1) * totB / G) - pl.b0;
  pl.c0 = (int)(c * totC / G);
  pl.nC = (int)((c + 1) * totC / G) - pl.c0;
  return pl;
}

__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                             ~(uintptr_t)127);
  float* red = reinterpret_cast<float*>(ring + kSlots * kSlotBytes);   // [2][kNg][kGw][32][4]
  __shared__ uint64_t full[kSlots], empty[kSlots];
  __shared__ int s_idx[kMaxR];          // expert of routed row t*k + j
  __shared__ float s_w[kMaxR];          // its weight
  __shared__ int s_roff[kMaxE + 1];     // rows of expert e: s_roff[e] .. s_roff[e+1]-1
  __shared__ int s_rows[kMaxR];         // sorted row -> routed row t*k + j
  __shared__ int s_inv[kMaxR];          // routed row -> sorted row
  __shared__ int s_tok[kMaxR];          // sorted row -> token
  __shared__ int s_act[kMaxE];          // active experts, increasing
  __shared__ int s_nact;
  __shared__ volatile int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.T, d = p.d, E = p.E, k = p.k, F = p.F;
  const int R = T * k;
  const int G = gridDim.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(smem_u32(full + i), 1);
      mbar_init(smem_u32(empty + i), kGw);
    }
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  pdl_wait();
  pdl_launch();
  __syncthreads();

  // ---------------------------------------------------------------- phase A
  if (warp < kCw) {
    // x -> fp16 (8 values per thread, all CTAs share the rows)
    const int n8 = T * d / 8;
    const uint4* xs = reinterpret_cast<const uint4*>(p.x);
    uint4* xo = reinterpret_cast<uint4*>(p.x16);
    for (int i = blockIdx.x * (kCw * 32) + threadIdx.x; i < n8; i += G * kCw * 32) {
      const uint4 v = xs[i];
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
      // stored as the pairs (e0,e4) (e1,e5) (e2,e6) (e3,e7), the K order of
      // the weight dequantisation
      uint32_t o[4];
      if (p.xf16) {
        // already fp16: pair the low (even j) or high (odd j) halves of
        // words j/2 and j/2 + 2
#pragma unroll
        for (int j = 0; j < 4; ++j)
          o[j] = __byte_perm(w4[j >> 1], w4[(j >> 1) + 2], (j & 1) ? 0x7632 : 0x5410);
      } else {
        float e[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          e[2 * j] = __uint_as_float(w4[j] << 16);
          e[2 * j + 1] = __uint_as_float(w4[j] & 0xFFFF0000u);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (!(fabsf(e[j]) < 65520.f && fabsf(e[j + 4]) < 65520.f))
            report_status(p.status, MOE_ERR_RANGE);
          asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(o[j]) : "f"(e[j + 4]), "f"(e[j]));
        }
      }
      xo[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    // router logits: a warp per (expert e, token t); per lane the 8-element
    // chunks lane, lane + 32, ... of the row in order, fp32 sums of exact
    // bf16 (or fp16) products, then a warp sum. All of a lane's chunks are loaded
    // before the first product.
    constexpr int kMaxC = 2048 / 256;          // 16-byte chunks per lane at d = 2048
    const int nc8 = d / 8;
    for (int u = blockIdx.x + G * warp; u < E * T; u += G * kCw) {
      const int e = u % E, t = u / E;
      const uint4* wrow = reinterpret_cast<const uint4*>(p.wr + (size_t)e * d);
      const uint4* xrow = reinterpret_cast<const uint4*>(p.x + (size_t)t * d);
      uint4 wv[kMaxC], xv[kMaxC];
#pragma unroll
      for (int i = 0; i < kMaxC; ++i) {
        const bool in = lane + 32 * i < nc8;
        wv[i] = in ? __ldg(wrow + lane + 32 * i) : make_uint4(0, 0, 0, 0);
        xv[i] = in ? xrow[lane + 32 * i] : make_uint4(0, 0, 0, 0);
      }
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < kMaxC; ++i) {
        if (lane + 32 * i < nc8) {
          const uint32_t wa[4] = {wv[i].x, wv[i].y, wv[i].z, wv[i].w};
          const uint32_t wb[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 fa = p.xf16 ? __half22float2(*reinterpret_cast<const __half2*>(&wa[q]))
                                     : bf16x2_to_f32x2(wa[q]);
            const float2 fb = p.xf16 ? __half22float2(*reinterpret_cast<const __half2*>(&wb[q]))
                                     : bf16x2_to_f32x2(wb[q]);
            acc = fmaf(fb.x, fa.x, acc);
            acc = fmaf(fb.y, fa.y, acc);
          }
        }
      }
      const float v = warp_sum(acc);
      if (lane == 0) p.logits[(size_t)t * E + e] = v + (p.rbias ? p.rbias[e] : 0.f);
    }
  }
  bool ok = true;
  if (warp < kCw) ok = grid_barrier(p.sync, 1, &s_abort, p.status, p.wait_limit);
  __syncthreads();
  if (s_abort) ok = false;

  // ---------------------------------------------------------------- routing
  if (ok && warp < kCw)
    for (int t = warp; t < T; t += kCw)
      topk_token(p.logits + (size_t)t * E, E, k, lane, s_idx + t * k, s_w + t * k);
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
    int rk = 0;
    if (threadIdx.x < R) rk = s_roff[s_idx[threadIdx.x]] + s_rows[threadIdx.x];
    __syncthreads();
    if (threadIdx.x < R) {
      s_rows[rk] = threadIdx.x;          // sorted row -> routed row
      s_inv[threadIdx.x] = rk;           // routed row -> sorted row
      s_tok[rk] = threadIdx.x / k;
    }
  }
  __syncthreads();
  const Plan pl = make_plan(d, F, p.gshift, s_nact);
  const int nseq = pl.nB + pl.nC;        // ring sequence of this CTA

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
            !mbar_wait(smem_u32(empty + slot), ((s / kSlots) - 1) & 1, &s_abort, p.status, true,
                       p.wait_limit))
          break;
        const uint32_t dst = smem_u32(ring + slot * kSlotBytes);
        const uint32_t bar = smem_u32(full + slot);
        // slot layout: 16 weight rows of K/2 bytes, then the 16 rows'
        // scales, then their biases
        if (s < pl.nB) {
          const int gi = pl.b0 + s;
          const int e = s_act[gi / pl.fpb], f0 = (gi % pl.fpb) * 8;
          const size_t rg = (size_t)e * 2 * F + f0, ru = rg + F;   // first gate / up row
          const uint32_t wb = 8u * (uint32_t)(d / 2), sb = 8u * 2u * (uint32_t)(d >> p.gshift);
          mbar_expect_tx(bar, 2 * wb + 4 * sb);
          bulk_g2s(dst, p.w_gu + rg * (d / 8), wb, bar);
          bulk_g2s(dst + wb, p.w_gu + ru * (d / 8), wb, bar);
          const uint32_t sc = dst + 2 * wb;
          const size_t gr = (size_t)(d >> p.gshift);          // groups per row
          bulk_g2s(sc, p.s_gu + rg * gr, sb, bar);
          bulk_g2s(sc + sb, p.s_gu + ru * gr, sb, bar);
          bulk_g2s(sc + 2 * sb, p.b_gu + rg * gr, sb, bar);
          bulk_g2s(sc + 3 * sb, p.b_gu + ru * gr, sb, bar);
        } else {
          const int di = pl.c0 + (s - pl.nB);
          const int a = di / pl.opb, ob = di % pl.opb;
          const size_t r = (size_t)s_act[a] * d + (size_t)ob * pl.dr;  // first of dr rows
          const uint32_t wb = (uint32_t)pl.dr * (uint32_t)(F / 2);
          const uint32_t sb = (uint32_t)pl.dr * 2u * (uint32_t)(F >> p.gshift);
          mbar_expect_tx(bar, wb + 2 * sb);
          bulk_g2s(dst, p.w_dn + r * (F / 8), wb, bar);
          const uint32_t sc = dst + wb;
          bulk_g2s(sc, p.s_dn + r * (size_t)(F >> p.gshift), sb, bar);
          bulk_g2s(sc + sb, p.b_dn + r * (size_t)(F >> p.gshift), sb, bar);
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
    // Lane (g, c) holds A rows g and g + 8 (gate row g and up row g of the 8
    // features, or output rows g and g + 8 of the 16) and token g of each
    // group of 8 (B columns). Each warp of a group multiplies its K steps;
    // the group adds the four partial sums in warp order (double-buffered
    // scratch, one group barrier per 8 tokens) and warp 0 of the group
    // stores the result.
    const int g = lane >> 2, c = lane & 3;
    const int grp = warp / kGw, gw = warp % kGw;
    int buf = 0;
    // sums the partials of warps gw .. gw + ks - 1 of the group into a4 (in
    // the first of them, gw % ks == 0)
    auto reduce = [&](const float* acc, float* a4, int ks) {
      float* rb = red + (((size_t)buf * kNg + grp) * kGw) * 128;
      *reinterpret_cast<float4*>(rb + gw * 128 + lane * 4) = make_float4(acc[0], acc[1], acc[2],
                                                                         acc[3]);
      group_sync(grp);
      a4[0] = a4[1] = a4[2] = a4[3] = 0.f;
      if (gw % ks == 0) {
        for (int w = gw; w < gw + ks; ++w) {
          const float4 v = *reinterpret_cast<const float4*>(rb + w * 128 + lane * 4);
          a4[0] += v.x;
          a4[1] += v.y;
          a4[2] += v.z;
          a4[3] += v.w;
        }
      }
      buf ^= 1;
    };

    // gate|up + SwiGLU -> h (fp16; every 8 features stored in the order
    // (0,4,1,5,2,6,3,7), the K order of the down projection's dequantisation)
    const int nstB = d / 128;
    const int rsB = d / 2;
    for (int s = grp; s < pl.nB; s += kNg) {
      const int slot = s % kSlots;
      ok = __all_sync(0xffffffffu, ok && mbar_wait(smem_u32(full + slot), (s / kSlots) & 1,
                                                   &s_abort, p.status, true, p.wait_limit));
      ok = group_sync_and(grp, ok);
      if (!ok) break;
      const uint8_t* sp = ring + slot * kSlotBytes;
      const int gi = pl.b0 + s;
      const int f0 = (gi % pl.fpb) * 8;
      const int e = s_act[gi / pl.fpb];
      const int r0 = s_roff[e], nv = s_roff[e + 1] - r0;
      const uint16_t* scl = reinterpret_cast<const uint16_t*>(sp + 16 * rsB);
      const int gB = d >> p.gshift;                // groups per row
      const uint16_t* sg = scl + g * gB;
      const uint16_t* su = scl + (8 + g) * gB;
      const uint16_t* bg = scl + (16 + g) * gB;
      const uint16_t* bu = scl + (24 + g) * gB;
      for (int q = 0; q * 8 < nv; ++q) {
        const int n = q * 8 + g;
        const bool xv = n < nv;
        const __half* xr = p.x16 + (size_t)(xv ? s_tok[r0 + n] : 0) * d;
        float acc[4], a4[4];
        warp_mma_steps(sp + g * rsB, sp + (8 + g) * rsB, sg, bg, su, bu, xr, xv, gw, nstB, kGw,
                       p.gshift, c, acc);
        reduce(acc, a4, kGw);
        // lane (g, c): gate (a4[0..1]) and up (a4[2..3]) of feature f0 + g
        // for the expert's tokens q*8 + 2c, q*8 + 2c + 1
        if (gw == 0) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int n2 = q * 8 + 2 * c + j;
            if (n2 < nv) {
              const float v = glu(p.act, a4[j], a4[2 + j]);
              if (!(fabsf(v) < 65520.f)) report_status(p.status, MOE_ERR_RANGE);
              p.h[(size_t)(r0 + n2) * F + f0 + (g & 3) * 2 + (g >> 2)] = __float2half_rn(v);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(empty + slot));
    }
    // all of h is written before any CTA reads it
    if (!grid_barrier(p.sync, 2, &s_abort, p.status, p.wait_limit)) ok = false;

    // down -> ys (fp16, sorted row order): an item is dr output rows of active
    // expert a against the expert's h rows; with 32 rows, warps 0-1 of the
    // group take rows 0-15 and warps 2-3 rows 16-31, each pair splitting K
    const int nstC = F / 128;
    const int rsC = F / 2;
    const int ksC = kGw / (pl.dr / 16);           // warps per 16 rows
    const int rbC = (gw / ksC) * 16;              // this warp's first row of the item
    for (int s = pl.nB + (((grp - pl.nB) % kNg) + kNg) % kNg; s < nseq; s += kNg) {
      const int slot = s % kSlots;
      ok = __all_sync(0xffffffffu, ok && mbar_wait(smem_u32(full + slot), (s / kSlots) & 1,
                                                   &s_abort, p.status, true, p.wait_limit));
      ok = group_sync_and(grp, ok);
      if (!ok) break;
      const uint8_t* sp = ring + slot * kSlotBytes;
      const int di = pl.c0 + (s - pl.nB);
      const int a = di / pl.opb, o0 = (di % pl.opb) * pl.dr + rbC;
      const int e = s_act[a];
      const int r0 = s_roff[e], nv = s_roff[e + 1] - r0;
      const uint16_t* sc_ = reinterpret_cast<const uint16_t*>(sp + pl.dr * rsC);
      const int gC = F >> p.gshift;                // groups per row
      const uint16_t* bi_ = sc_ + pl.dr * gC;
      const int ra = rbC + g, rb_ = rbC + 8 + g;     // A rows g and g + 8 of this warp
      for (int q = 0; q * 8 < nv; ++q) {
        const int n = q * 8 + g;
        const bool hvld = n < nv;
        const __half* hr = p.h + (size_t)(hvld ? r0 + n : 0) * F;
        float acc[4], a4[4];
        warp_mma_steps(sp + ra * rsC, sp + rb_ * rsC, sc_ + ra * gC, bi_ + ra * gC, sc_ + rb_ * gC,
                       bi_ + rb_ * gC, hr, hvld, gw % ksC, nstC, ksC, p.gshift, c, acc);
        reduce(acc, a4, ksC);
        // lane (g, c): outputs o0 + g (a4[0..1]) and o0 + 8 + g (a4[2..3])
        // of the expert's rows q*8 + 2c, q*8 + 2c + 1
        if (gw % ksC == 0) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int n2 = q * 8 + 2 * c + j;
            if (n2 < nv) {
              if (!(fabsf(a4[j]) < 65520.f && fabsf(a4[2 + j]) < 65520.f))
                report_status(p.status, MOE_ERR_RANGE);
              __half* yr = p.ys + (size_t)(r0 + n2) * d + o0;
              yr[g] = __float2half_rn(a4[j]);
              yr[g + 8] = __float2half_rn(a4[2 + j]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(empty + slot));
    }
    // all of ys is written before any CTA reads it
    if (!grid_barrier(p.sync, 3, &s_abort, p.status, p.wait_limit)) ok = false;

    // combine: y[t][o .. o+7] = sum over j of w[t][j] * ys[inv[t*k + j]][o ..
    // o+7], fp32 fused multiply-adds in j order, one rounding to bf16 (fp16)
    if (ok) {
      const int per_row = d / 8;
      for (int i = blockIdx.x * (kCw * 32) + threadIdx.x; i < T * per_row; i += G * kCw * 32) {
        const int t = i / per_row, o = (i % per_row) * 8;
        float acc8[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc8[q] = 0.f;
        for (int j = 0; j < k; ++j) {
          const float wj = s_w[t * k + j];
          const uint4 v = __ldcg(reinterpret_cast<const uint4*>(
              p.ys + (size_t)s_inv[t * k + j] * d + o));
          const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[q]));
            acc8[2 * q] = fmaf(wj, f.x, acc8[2 * q]);
            acc8[2 * q + 1] = fmaf(wj, f.y, acc8[2 * q + 1]);
          }
        }
        uint4 out;
        if (p.xf16) {
          uint32_t o4[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const __half2 hq = __floats2half2_rn(acc8[2 * q], acc8[2 * q + 1]);
            o4[q] = *reinterpret_cast<const uint32_t*>(&hq);
          }
          out = make_uint4(o4[0], o4[1], o4[2], o4[3]);
        } else {
          out.x = pack_bf16x2(acc8[0], acc8[1]);
          out.y = pack_bf16x2(acc8[2], acc8[3]);
          out.z = pack_bf16x2(acc8[4], acc8[5]);
          out.w = pack_bf16x2(acc8[6], acc8[7]);
        }
        *reinterpret_cast<uint4*>(p.y + (size_t)t * d + o) = out;
      }
    }
  }

  // the workspace tables, as moe_route and moe_sort_rows write them, by the
  // last CTA once its own work is done: they are not needed inside this
  // launch
  if (!s_abort && blockIdx.x == G - 1) {
    for (int i = threadIdx.x; i < R; i += kThreads) {
      p.topk_idx[i] = s_idx[i];
      p.topk_w[i] = s_w[i];
      p.order[i] = (uint32_t)s_rows[i];
      p.inv_order[i] = (uint32_t)s_inv[i];
      p.row_map[i] = (uint32_t)(s_rows[i] / k);
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
}

// Test support: each kind of bounded wait of this file, made to run out. The
// mbarrier expects two arrivals and gets one; the grid barrier of a one-CTA
// grid waits for arrivals number 1 and 2 of barrier 2 after only one. Both
// must give up after `limit` cycles, record MOE_ERR_TIMEOUT and return.
__global__ void __launch_bounds__(kThreads, 1) wait_selftest_kernel(int which, long long limit,
                                                                    unsigned* ctr, int* status) {
  __shared__ uint64_t bar;
  __shared__ volatile int s_abort;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 2);
    s_abort = 0;
    *ctr = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    __threadfence();
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  if (which == 1) {
    if (threadIdx.x == 0) {
      mbar_arrive(smem_u32(&bar));
      mbar_wait(smem_u32(&bar), 0, &s_abort, status, true, limit);
    }
  } else if (warp < kCw) {
    grid_barrier(ctr, 2, &s_abort, status, limit);
  }
  __syncthreads();
}

// ------------------------------------------------------------------ host

static int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

}  // namespace dec

cudaError_t launch_decode_wait_selftest(int which, long long limit, unsigned* ctr, int* status,
                                        cudaStream_t s) {
  dec::wait_selftest_kernel<<<1, dec::kThreads, 0, s>>>(which, limit, ctr, status);
  return cudaGetLastError();
}

bool decode_fused_ok(int T, int k, int E, int d, int F, int fmt, int dt) {
  using namespace dec;
  return q4_group(fmt) != 0 && (dt == MOE_BF16 || dt == MOE_F16) && T >= 1 && T <= kMaxT && T * k <= kMaxR &&
         E <= kMaxE && k <= 32 && d % 128 == 0 && F % 128 == 0 && d <= 2048 && F <= 2048;
}

size_t decode_smem_bytes() { return dec::kSlots * dec::kSlotBytes + dec::kRedBytes + 128; }

cudaError_t launch_decode_fused(const void* x, int dt, const void* w_router, const float* bias,
                                const moe_experts& ex, int T, int k, int BM, float* logits,
                                int32_t* idx, float* w, uint32_t* order, uint32_t* inv_order,
                                uint32_t* row_map, int32_t* counts, int32_t* row_off,
                                int32_t* tile_off, void* x16, void* h, void* ys, void* y,
                                unsigned* sync, int* status, cudaStream_t s) {
  using namespace dec;
  if (!decode_fused_ok(T, k, ex.E, ex.d, ex.F, ex.fmt, dt)) return cudaErrorNotSupported;
  const int G = sm_count();
  if (G <= 0) return cudaErrorNoDevice;
  Params p{};
  p.x = (const uint16_t*)x;
  p.wr = (const uint16_t*)w_router;
  p.xf16 = dt == MOE_F16;
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
  p.act = ex.act;
  p.gs = q4_group(ex.fmt);
  p.gshift = p.gs == 32 ? 5 : p.gs == 64 ? 6 : 7;
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
  p.ys = (__half*)ys;
  p.y = (uint16_t*)y;
  p.sync = sync;
  p.status = status;
  p.wait_limit = wait_cycles();
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
