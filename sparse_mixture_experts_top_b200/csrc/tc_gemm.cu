// Tensor-core grouped GEMMs for the prefill regime (tcgen05 / TMEM / TMA).
//
// DS4Server issue #112, "Kernel contract": work is split into tiles that own
// sorted rows of one expert, found from per-expert tile and row prefix tables
// by binary search; gate|up reads token rows in place through row_map and
// writes silu(gate) * up; the down projection reads rows already sorted by
// expert. mlx-lm PR #2044, "What": each expert's weights are read and
// dequantised once per tile instead of once per (token, slot).
//
// B200 design (one persistent CTA per SM, 16 warps):
//   * swap-AB: the MMA's M = 128 weight rows (output features), N = the
//     tile's token rows (<= 128, rounded up to 16 per tile at run time), so
//     a tile with few rows costs proportionally few tensor cycles;
//   * warp 0: TMA loads of the raw weight tile (packed q4 words or bf16,
//     128-byte rows) into a shared-memory ring;
//   * warp 2: cp.async copies of the tile's token rows -- through row_map
//     (gather) or contiguous -- into a 128B-swizzled K-major ring (per-row
//     TMA loads cost ~30 ns of issue each, which starved the tensor core);
//   * warps 8..15 (dequant): each thread owns one weight row (one TMEM lane):
//     reads its packed words from shared memory, dequantises w = s*q + b to
//     bf16 pairs and writes them into TMEM with tcgen05.st, where the MMA
//     takes them as its A operand -- the dequantised tile never goes back
//     through shared memory;
//   * warp 1 (MMA): one thread issues tcgen05.mma (A from TMEM, B from
//     shared memory) into fp32 accumulators in TMEM; gate and up accumulate
//     side by side so one token tile feeds both;
//   * warps 4..7 (epilogue): tcgen05.ld of the accumulators, SwiGLU to fp16
//     (gate|up) or an fp32 store (down projection; router logits + bias).
// The expert GEMMs multiply fp16 operands (x converted once from bf16,
// weights dequantised to fp16, h stored in fp16): 11-bit operands keep the
// rounding of the dequantised weights and of h 8x below bf16's; values
// outside the fp16 range are reported as MOE_ERR_RANGE. The router keeps its
// bf16 operands, which are exact there.
// Every mbarrier wait is bounded (about a second): on expiry the kernel
// records MOE_ERR_TIMEOUT in the status word, all roles leave their loops,
// copies in flight are waited for (bounded), TMEM is freed, and it returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace moe {
namespace tc {

constexpr int BN = 128;        // token rows per tile (the sort tables' BM)
constexpr int BMW = 128;       // weight rows per tile (MMA M)
constexpr int KA = 64;         // K elements per A stage (one q4 group)
constexpr int kMaxE = 1024;    // tile / row tables cached in shared memory
constexpr int kThreads = 512;
constexpr int kEpiWarp0 = 4;
constexpr int kDqWarp0 = 8;
constexpr long long kWaitCycles = 2000000000LL;   // ~1 s at the B200's clocks

enum { EPI_SWIGLU = 0, EPI_STORE_F32 = 1 };   // fp32 store adds p.bias when set

template <int FMT, int EPI>
struct Cfg {
  static constexpr int NMAT = EPI == EPI_SWIGLU ? 2 : 1;
  static constexpr bool Q4 = FMT == MOE_W_Q4G64;
  static constexpr int KR = Q4 ? 256 : 64;                  // K elements per raw stage
  static constexpr int RAW_ROW = 128;                       // bytes per weight row per raw stage
  static constexpr int RAW_MAT = BMW * RAW_ROW;
  static constexpr int RAW_BYTES = NMAT * RAW_MAT;
  static constexpr int A_PER_RAW = KR / KA;                 // 4 (q4) or 1 (bf16)
#ifndef MOE_TC_RAW_KB
#define MOE_TC_RAW_KB 96
#endif
  static constexpr int NR_FIT = (MOE_TC_RAW_KB * 1024) / RAW_BYTES;
  static constexpr int NR = NR_FIT > 8 ? 8 : NR_FIT;
  static constexpr int ACC_COLS = NMAT * BN;
  static constexpr int A_COLS = NMAT * (KA / 2);            // 32-bit TMEM columns per A stage
  // k-block stages: stage s = A slot s (TMEM) + B slot s (shared memory).
  // The MMA releases stages in pairs (one commit per two k-blocks: each
  // tcgen05.commit costs the tensor pipe ~200 cycles), so NS is even.
  static constexpr int NS = NMAT == 2 ? 4 : 6;
  static constexpr int B_BYTES = BN * 128;
  // warps that write one A stage: NMAT == 2: 4 gate + 4 up warps;
  // NMAT == 1: q4 -- the 4 warps of one half of the raw row; bf16 -- all 8
  // (half the columns each)
  static constexpr int A_ARRIVALS = NMAT == 2 ? 8 : (Q4 ? 4 : 8);
  // q4 scales and biases of a raw stage: [NMAT][128 rows][4 groups] bf16 each
  static constexpr int SCL_BYTES = Q4 ? NMAT * BMW * 4 * 2 * 2 : 0;
  static constexpr int TABLES = 2 * (kMaxE + 1) * 4 + BN * 4;  // tile/row tables, tile rows
  static_assert(NS % 2 == 0 && ACC_COLS + NS * A_COLS <= 512, "stages must fit TMEM in pairs");
  static constexpr int SMEM = 1024 + NR * RAW_BYTES + NS * B_BYTES + 1024 + TABLES + NR * SCL_BYTES;
};

struct Params {
  const int32_t* row_off;
  const int32_t* tile_off;
  int E;               // groups (experts); 1 for the router
  int n_rows;          // router: tokens T
  int n_mb;            // weight-row blocks per group
  int K;               // reduction length
  int rows_per_group;  // weight rows per expert in the stacked tensor
  int up_off;          // row offset of the up matrix inside an expert
  int G;               // q4 groups per weight row (K / 64)
  const uint16_t* scales;
  const uint16_t* biases;
  const uint32_t* row_map;  // token of each sorted row (gather), or null
  const void* b_src;        // token rows: [rows][K] 16-bit (x16, h or x)
  void* out;
  int out_ld;          // elements per output row
  int m_limit;         // valid weight rows per group (router: E)
  const float* bias;   // router bias or null
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
__device__ __forceinline__ void mbar_arrive_tx(uint32_t bar, uint32_t bytes) {
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

// Bounded wait for the phase of `parity` to complete. Returns false when the
// kernel is aborting (another role timed out) or this wait ran out.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int* status, bool honor_abort = true) {
  if (mbar_try(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try(bar, parity)) return true;
    if ((i & 63u) == 0) {
      if (honor_abort && *abort_flag) return false;
      if (clock64() - t0 > kWaitCycles) {
        *abort_flag = 1;
        report_status(status, MOE_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Every lane waits; the result is the same in all lanes, so the warp stays
// converged for the .sync.aligned tcgen05 instructions that follow.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity,
                                               volatile int* abort_flag, int* status) {
  const bool r = mbar_wait(bar, parity, abort_flag, status);
  return __all_sync(0xffffffffu, r);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* tm, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16 (bf16 in, fp32 accumulate)
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
      "r"(a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// The MMAs of one 64-deep k-block (4 K-steps of 16) for one or two
// accumulators, in a single statement: A columns a (+8 per K-step), B
// descriptor low word blo (+2 per K-step, i.e. +32 bytes inside the 128-byte
// swizzle atom), accumulate unless `first`. Keeping the issue path to a few
// instructions per MMA matters: the tensor core takes a K=16 step of an
// M=128 tile in ~80 cycles, and the single issuing thread must keep up.
__device__ __forceinline__ void mma_kblock2(uint32_t d0, uint32_t d1, uint32_t a0, uint32_t a1,
                                            uint32_t blo, uint32_t bhi, uint32_t idesc,
                                            uint32_t first) {
  asm volatile(
      "{\n\t.reg .pred pf, pt;\n\t.reg .b64 b0, b1, b2, b3;\n\t"
      "setp.eq.b32 pf, %7, 0;\n\t"
      "setp.ne.b32 pt, %6, 0;\n\t"
      "mov.b64 b0, {%4, %5};\n\t"
      "add.u32 %4, %4, 2;\n\tmov.b64 b1, {%4, %5};\n\t"
      "add.u32 %4, %4, 2;\n\tmov.b64 b2, {%4, %5};\n\t"
      "add.u32 %4, %4, 2;\n\tmov.b64 b3, {%4, %5};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%2], b0, %6, pf;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%1], [%3], b0, %6, pf;\n\t"
      "add.u32 %2, %2, 8;\n\tadd.u32 %3, %3, 8;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%2], b1, %6, pt;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%1], [%3], b1, %6, pt;\n\t"
      "add.u32 %2, %2, 8;\n\tadd.u32 %3, %3, 8;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%2], b2, %6, pt;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%1], [%3], b2, %6, pt;\n\t"
      "add.u32 %2, %2, 8;\n\tadd.u32 %3, %3, 8;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%2], b3, %6, pt;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%1], [%3], b3, %6, pt;\n\t}\n"
      : "+r"(d0), "+r"(d1), "+r"(a0), "+r"(a1), "+r"(blo), "+r"(bhi)
      : "r"(idesc), "r"(first)
      : "memory");
}
__device__ __forceinline__ void mma_kblock1(uint32_t d0, uint32_t a0, uint32_t blo, uint32_t bhi,
                                            uint32_t idesc, uint32_t first) {
  asm volatile(
      "{\n\t.reg .pred pf, pt;\n\t.reg .b64 b0, b1, b2, b3;\n\t"
      "setp.eq.b32 pf, %5, 0;\n\t"
      "setp.ne.b32 pt, %4, 0;\n\t"
      "mov.b64 b0, {%2, %3};\n\t"
      "add.u32 %2, %2, 2;\n\tmov.b64 b1, {%2, %3};\n\t"
      "add.u32 %2, %2, 2;\n\tmov.b64 b2, {%2, %3};\n\t"
      "add.u32 %2, %2, 2;\n\tmov.b64 b3, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], b0, %4, pf;\n\t"
      "add.u32 %1, %1, 8;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], b1, %4, pt;\n\t"
      "add.u32 %1, %1, 8;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], b2, %4, pt;\n\t"
      "add.u32 %1, %1, 8;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], b3, %4, pt;\n\t}\n"
      : "+r"(d0), "+r"(a0), "+r"(blo), "+r"(bhi)
      : "r"(idesc), "r"(first)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// K-major operand in shared memory, 128-byte swizzle, rows of 128 bytes,
// 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1 << 16;              // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;    // stride byte offset
  d |= (uint64_t)1 << 46;              // descriptor version for sm_100
  d |= (uint64_t)2 << 61;              // SWIZZLE_128B
  return d;
}

// M = 128, N = n, fp32 accumulate, both operands K-major; operand format
// fp16 (code 0) or bf16 (code 1)
__device__ __forceinline__ uint32_t idesc_mma(int n, bool f16) {
  const uint32_t ab = f16 ? 0u : 1u;
  return (1u << 4) | (ab << 7) | (ab << 10) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(BMW >> 4) << 24);
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------------ dequant

__device__ __forceinline__ uint32_t f16x2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t f16x2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
// (lo, hi) floats -> packed fp16 pair, lo in the low half, round to nearest
__device__ __forceinline__ uint32_t f16x2_pack(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}
// a bf16 value (low 16 bits of v) as an fp16 pair holding it twice
__device__ __forceinline__ uint32_t f16x2_from_bf16(uint32_t v) {
  const float f = __uint_as_float(v << 16);
  return f16x2_pack(f, f);
}
// two bf16 values (element 2c low, 2c+1 high) -> the same pair in fp16
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
  return f16x2_pack(__uint_as_float(v << 16), __uint_as_float(v & 0xFFFF0000u));
}

// 8 nibbles of one word (element j in bits [4j, 4j+3]) -> 4 fp16 pairs
// (element 2c in the low half of out[c]), value = s * q + b rounded once.
// Each nibble q is placed in the mantissa of fp16 1024.0 (0x6400 | q =
// 1024 + q, exact), 1024 is subtracted exactly, then one fused multiply-add
// applies the group's scale and bias (s2, b2: fp16 pairs).
__device__ __forceinline__ void dequant_word(uint32_t w, uint32_t s2, uint32_t b2, uint32_t* out) {
  const uint32_t lo = w & 0x0F0F0F0Fu;           // elements 0, 2, 4, 6
  const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;    // elements 1, 3, 5, 7
  const uint32_t p0 = __byte_perm(lo, hi, 0x5140);   // e0 e1 e2 e3
  const uint32_t p1 = __byte_perm(lo, hi, 0x7362);   // e4 e5 e6 e7
  const uint32_t M = 0x64646464u;
  const uint32_t c1024 = 0x64006400u;
  out[0] = f16x2_fma(f16x2_sub(__byte_perm(p0, M, 0x4140), c1024), s2, b2);
  out[1] = f16x2_fma(f16x2_sub(__byte_perm(p0, M, 0x4342), c1024), s2, b2);
  out[2] = f16x2_fma(f16x2_sub(__byte_perm(p1, M, 0x4140), c1024), s2, b2);
  out[3] = f16x2_fma(f16x2_sub(__byte_perm(p1, M, 0x4342), c1024), s2, b2);
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// ------------------------------------------------------------------ tiles

// Tile tau -> (expert e, first sorted row r0, valid rows nv), with the
// prefix tables read from their shared-memory copies.
template <bool ROUTER>
__device__ __forceinline__ void decode_tile(const Params& p, const int* s_toff, const int* s_roff,
                                            int u, int& e, int& mb, int& r0, int& nv) {
  const int tau = u / p.n_mb;
  mb = u - tau * p.n_mb;
  if (ROUTER) {
    e = 0;
    r0 = tau * BN;
    nv = min(BN, p.n_rows - r0);
  } else {
    int lo = 0, hi = p.E - 1;      // largest e with tile_off[e] <= tau
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_toff[mid] <= tau) lo = mid; else hi = mid - 1;
    }
    e = lo;
    r0 = s_roff[e] + (tau - s_toff[e]) * BN;
    nv = min(BN, s_roff[e + 1] - r0);
  }
}

template <bool ROUTER>
__device__ __forceinline__ int total_units(const Params& p, const int* s_toff) {
  if (ROUTER) return ((p.n_rows + BN - 1) / BN) * p.n_mb;
  return s_toff[p.E] * p.n_mb;
}

// ------------------------------------------------------------------ kernel

template <int FMT, int EPI, bool GATHER, bool ROUTER>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_tc_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tmA) {
  pdl_wait();
  pdl_launch();
  using C = Cfg<FMT, EPI>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  const uint32_t raw_base = smem_u32(smem);
  const uint32_t b_base = raw_base + C::NR * C::RAW_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::NR * C::RAW_BYTES + C::NS * C::B_BYTES);
  uint64_t* raw_full = bars;
  uint64_t* raw_empty = raw_full + C::NR;
  uint64_t* a_full = raw_empty + C::NR;
  uint64_t* b_full = a_full + C::NS;
  uint64_t* s_empty = b_full + C::NS;    // [NS / 2]: stage pair released by the MMA
  uint64_t* acc_full = s_empty + C::NS / 2;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_toff = reinterpret_cast<int*>(smem + C::NR * C::RAW_BYTES + C::NS * C::B_BYTES + 1024);
  int* s_roff = s_toff + kMaxE + 1;
  int* s_trow = s_roff + kMaxE + 1;     // [BN] source rows of the loader's current tile
  // q4 scale ring: raw stage rs holds scales [NMAT][128][4] then biases [NMAT][128][4]
  const uint32_t scl_base = smem_u32(s_trow + BN);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NR; ++i) {
      // q4: the TMA arrive + the 32 lanes' cp.async arrivals for the scales
      mbar_init(smem_u32(raw_full + i), C::Q4 ? 33 : 1);
      mbar_init(smem_u32(raw_empty + i), 8);
    }
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(smem_u32(a_full + i), C::A_ARRIVALS);
      mbar_init(smem_u32(b_full + i), 32);  // the loader's 32 lanes, as their copies land
    }
    for (int i = 0; i < C::NS / 2; ++i) mbar_init(smem_u32(s_empty + i), 1);
    mbar_init(smem_u32(acc_full), 1);
    mbar_init(smem_u32(acc_empty), 4);
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     smem_u32(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // the prologue above overlaps the previous kernel; everything below reads
  // what earlier kernels wrote
  pdl_wait();
  pdl_launch();
  if (!ROUTER) {
    for (int i = threadIdx.x; i <= p.E; i += blockDim.x) {
      s_toff[i] = __ldg(p.tile_off + i);
      s_roff[i] = __ldg(p.row_off + i);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int total = total_units<ROUTER>(p, s_toff);
  const int nkr = p.K / C::KR;           // raw stages per tile
  const int nka = p.K / KA;              // A stages per tile

  if (warp == 0) {
    // ------------------------------------------------------------ raw weights (TMA)
    uint32_t raw_it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
      int e, mb, r0, nv;
      decode_tile<ROUTER>(p, s_toff, s_roff, u, e, mb, r0, nv);
      const int wrow = (ROUTER ? 0 : e * p.rows_per_group) + mb * BMW;
      for (int kr = 0; kr < nkr && ok; ++kr) {
        const int rs = raw_it % C::NR;
        ok = mbar_wait_warp(smem_u32(raw_empty + rs), ((raw_it / C::NR) & 1) ^ 1, abort_flag,
                            p.status);
        if (!ok) break;
        if (C::Q4) {
          // the stage's scales and biases (4 groups of each weight row), 8
          // bytes per row and array, copied by the 32 lanes; each lane's
          // arrival fires when its copies have landed
          const uint32_t sdst = scl_base + rs * C::SCL_BYTES;
#pragma unroll
          for (int mat = 0; mat < C::NMAT; ++mat)
#pragma unroll
            for (int j = 0; j < BMW / 32; ++j) {
              const int m = lane + 32 * j;
              const size_t grow = (size_t)wrow + (mat ? p.up_off : 0) + m;
              const uint32_t o = (uint32_t)((mat * BMW + m) * 8);
              asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(sdst + o),
                           "l"(p.scales + grow * p.G + 4 * kr)
                           : "memory");
              asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(
                               sdst + C::SCL_BYTES / 2 + o),
                           "l"(p.biases + grow * p.G + 4 * kr)
                           : "memory");
            }
          asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(
                           smem_u32(raw_full + rs))
                       : "memory");
        }
        if (lane == 0) {
          const uint32_t dst = raw_base + rs * C::RAW_BYTES;
          const uint32_t bar = smem_u32(raw_full + rs);
          const int x = kr * (C::Q4 ? C::KR / 8 : C::KR);
          mbar_arrive_tx(bar, C::RAW_BYTES);
          tma_load_2d(dst, &tmA, x, wrow, bar);
          if (C::NMAT == 2) tma_load_2d(dst + C::RAW_MAT, &tmA, x, wrow + p.up_off, bar);
        }
        ++raw_it;
      }
    }
    // copies in flight: wait (bounded, also when aborting) for the last
    // phase issued on every stage before the CTA may exit
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (lane == 0) {
      for (uint32_t i = 0; i < (uint32_t)C::NR && i < raw_it; ++i) {
        const uint32_t last = raw_it - 1 - i;
        mbar_wait(smem_u32(raw_full + last % C::NR), (last / C::NR) & 1, abort_flag, p.status, false);
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------ token rows (cp.async)
    // Lane l copies 16-byte chunks l, l + 32, ... of the tile's rows (chunk c
    // of row n lands at n*128 + ((c ^ (n & 7)) * 16): the 128B-swizzled
    // K-major layout the MMA reads). Each lane then arms a hardware arrival
    // on the stage's barrier that fires once its copies have landed, so the
    // loader never waits for its own copies; the MMA thread, after the
    // barrier, fences the async proxy before the tensor core reads them.
    const uint16_t* src = reinterpret_cast<const uint16_t*>(p.b_src);
    uint32_t b_it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
      int e, mb, r0, nv;
      decode_tile<ROUTER>(p, s_toff, s_roff, u, e, mb, r0, nv);
      __syncwarp();
      for (int n = lane; n < nv; n += 32) s_trow[n] = GATHER ? (int)__ldg(p.row_map + r0 + n) : r0 + n;
      __syncwarp();
      for (int kb = 0; kb < nka && ok; ++kb) {
        const int bs = b_it % C::NS;
        ok = mbar_wait_warp(smem_u32(s_empty + (bs >> 1)), ((b_it / C::NS) & 1) ^ 1, abort_flag,
                            p.status);
        if (!ok) break;
        const uint32_t dst = b_base + bs * C::B_BYTES;
        for (int i = lane; i < nv * 8; i += 32) {
          const int n = i >> 3, c = i & 7;
          const uint16_t* g = src + (size_t)s_trow[n] * p.K + kb * KA + c * 8;
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                           dst + n * 128 + ((c ^ (n & 7)) << 4)),
                       "l"(g)
                       : "memory");
        }
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(
                         smem_u32(b_full + bs))
                     : "memory");
        ++b_it;
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t tcount = 0;
      uint32_t ss = 0, sph = 0;                       // stage slot and its phase
      bool ok = true;
      // descriptor of B stage 0 (low word: start address / 16 and the
      // leading offset; high word: stride offset, version, swizzle)
      const uint64_t d0 = desc_sw128(b_base);
      const uint32_t blo0 = (uint32_t)d0, bhi = (uint32_t)(d0 >> 32);
      const uint32_t a_col0 = tmem + C::ACC_COLS;
      for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
        int e, mb, r0, nv;
        decode_tile<ROUTER>(p, s_toff, s_roff, u, e, mb, r0, nv);
        const int n_mma = max(16, (nv + 15) & ~15);
        const uint32_t idesc = idesc_mma(n_mma, !ROUTER);
        if (tcount > 0) {
          ok = mbar_wait(smem_u32(acc_empty), (tcount - 1) & 1, abort_flag, p.status);
          if (!ok) break;
          tc_fence_after();
        }
        for (int kb = 0; kb < nka && ok; ++kb) {
          ok = mbar_wait(smem_u32(a_full + ss), sph, abort_flag, p.status) &&
               mbar_wait(smem_u32(b_full + ss), sph, abort_flag, p.status);
          if (!ok) break;
          // the token rows were written by cp.async (generic proxy); the
          // tensor core reads them through the async proxy
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          tc_fence_after();
          const uint32_t blo = blo0 + ss * (uint32_t)(C::B_BYTES >> 4);
          const uint32_t acol = a_col0 + ss * (uint32_t)C::A_COLS;
          if (C::NMAT == 2)
            mma_kblock2(tmem, tmem + BN, acol, acol + KA / 2, blo, bhi, idesc, kb == 0);
          else
            mma_kblock1(tmem, acol, blo, bhi, idesc, kb == 0);
          // K is a multiple of 128, so a tile has an even number of
          // k-blocks and the pairs never straddle tiles
          if (ss & 1) mma_commit(smem_u32(s_empty + (ss >> 1)));
          if (++ss == (uint32_t)C::NS) { ss = 0; sph ^= 1; }
        }
        if (!ok) break;
        mma_commit(smem_u32(acc_full));
        ++tcount;
      }
      // all MMAs issued by this thread complete before TMEM is released
      mma_commit(smem_u32(drain));
      mbar_wait(smem_u32(drain), 0, abort_flag, p.status, false);
    }
    __syncwarp();
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int m = q * 32 + lane;                      // weight row of this thread
    const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
    uint32_t tcount = 0;
    bool range_ok = true;
    for (int u = blockIdx.x; u < total; u += gridDim.x) {
      int e, mb, r0, nv;
      decode_tile<ROUTER>(p, s_toff, s_roff, u, e, mb, r0, nv);
      if (!mbar_wait_warp(smem_u32(acc_full), tcount & 1, abort_flag, p.status)) break;
      tc_fence_after();
      const int orow = mb * BMW + m;                  // output feature
      const bool mok = orow < p.m_limit;
      for (int c0 = 0; c0 < nv; c0 += 16) {
        uint32_t g[16];
        tmem_ld16(tl + c0, g);
        if (EPI == EPI_SWIGLU) {
          uint32_t uu[16];
          tmem_ld16(tl + BN + c0, uu);
          tmem_ld_wait();
          __half* h = reinterpret_cast<__half*>(p.out);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = c0 + j;
            if (n < nv) {
              const float v = swiglu(__uint_as_float(g[j]), __uint_as_float(uu[j]));
              range_ok &= fabsf(v) < 65520.f;    // rounds to a finite fp16
              h[(size_t)(r0 + n) * p.out_ld + orow] = __float2half_rn(v);
            }
          }
        } else {
          tmem_ld_wait();
          float* o = reinterpret_cast<float*>(p.out);
          const float bv = (mok && p.bias) ? __ldg(p.bias + orow) : 0.f;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = c0 + j;
            if (n < nv && mok) o[(size_t)(r0 + n) * p.out_ld + orow] = __uint_as_float(g[j]) + bv;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(acc_empty));
      ++tcount;
    }
    if (!__all_sync(0xffffffffu, range_ok) && lane == 0) report_status(p.status, MOE_ERR_RANGE);
  } else if (warp >= kDqWarp0) {
    // ------------------------------------------------------------ dequant
    const int dw = warp - kDqWarp0;                   // 0..7
    const int q = warp & 3;                           // TMEM lane quadrant
    const int m = q * 32 + lane;                      // weight row of this thread
    const int part = dw >> 2;                         // matrix (NMAT 2) or half (NMAT 1)
    const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
    uint32_t raw_it = 0, a_it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
      int e, mb, r0, nv;
      decode_tile<ROUTER>(p, s_toff, s_roff, u, e, mb, r0, nv);
      for (int kr = 0; kr < nkr && ok; ++kr) {
        const int rs = raw_it % C::NR;
        ok = mbar_wait_warp(smem_u32(raw_full + rs), (raw_it / C::NR) & 1, abort_flag, p.status);
        if (!ok) break;
        const uint32_t rbase = raw_base + rs * C::RAW_BYTES;
        uint32_t vals[32];
        // q4: this row's 4 groups of scales and biases (bf16 pairs)
        uint32_t sc[2] = {0, 0}, bi[2] = {0, 0};
        if (C::Q4) {
          const uint32_t so = scl_base + rs * C::SCL_BYTES +
                              (uint32_t)(((C::NMAT == 2 ? part : 0) * BMW + m) * 8);
          asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(sc[0]), "=r"(sc[1]) : "r"(so));
          asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];"
                       : "=r"(bi[0]), "=r"(bi[1])
                       : "r"(so + C::SCL_BYTES / 2));
          if (C::NMAT == 1 && part) {   // half 1: groups 2, 3
            sc[0] = sc[1];
            bi[0] = bi[1];
          }
        }
        if (C::Q4) {
          // my row: 128 bytes = 8 chunks of 16 B (128-byte swizzle): chunk pair
          // (2j, 2j+1) holds the 64 elements of A stage j (group 4kr + j).
          // NMAT 2: this thread converts all 4 A stages of its matrix;
          // NMAT 1: half `part` converts A stages 2*part and 2*part + 1.
          const uint32_t rowa = rbase + (C::NMAT == 2 ? part * C::RAW_MAT : 0) + m * 128;
          const int sw = m & 7;
          constexpr int nst = C::NMAT == 2 ? 4 : 2;    // A stages this thread converts
          const int cbase = C::NMAT == 2 ? 0 : 4 * part;  // its first 16-byte chunk
          uint4 wv[2 * nst];
#pragma unroll
          for (int c = 0; c < 2 * nst; ++c) wv[c] = lds128(rowa + (((cbase + c) ^ sw) << 4));
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(raw_empty + rs));
#pragma unroll
          for (int st = 0; st < nst; ++st) {
            if (!ok) break;
            const int j = (C::NMAT == 2 ? 0 : 2 * part) + st;   // A stage within the raw stage
            const uint32_t sv = C::NMAT == 2 ? sc[st >> 1] : sc[0];
            const uint32_t bv = C::NMAT == 2 ? bi[st >> 1] : bi[0];
            const uint32_t s2 = f16x2_from_bf16((st & 1) ? (sv >> 16) : (sv & 0xFFFFu));
            const uint32_t b2 = f16x2_from_bf16((st & 1) ? (bv >> 16) : (bv & 0xFFFFu));
            const uint4 w0 = wv[2 * st], w1 = wv[2 * st + 1];
            const uint32_t ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) dequant_word(ws[i], s2, b2, vals + 4 * i);
            const uint32_t stage = a_it + j;
            const int as = stage % C::NS;
            ok = mbar_wait_warp(smem_u32(s_empty + (as >> 1)), ((stage / C::NS) & 1) ^ 1, abort_flag,
                                p.status);
            if (!ok) break;
            tc_fence_after();
            const uint32_t col = C::ACC_COLS + as * C::A_COLS + (C::NMAT == 2 ? part * (KA / 2) : 0);
            tmem_st16(tl + col, vals);
            tmem_st16(tl + col + 16, vals + 16);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(a_full + as));
          }
        } else {
          // bf16 weights: my row is 128 bytes = 8 chunks of 16 B, 128-byte swizzle
          const uint32_t rowa = rbase + (C::NMAT == 2 ? part * C::RAW_MAT : 0) + m * 128;
          const int sw = m & 7;
          const int c0 = C::NMAT == 2 ? 0 : 4 * part;
          const int nc = C::NMAT == 2 ? 8 : 4;
          for (int c = 0; c < nc; ++c) {
            const uint4 v = lds128(rowa + (((c0 + c) ^ sw) << 4));
            if (ROUTER) {
              vals[4 * c + 0] = v.x;
              vals[4 * c + 1] = v.y;
              vals[4 * c + 2] = v.z;
              vals[4 * c + 3] = v.w;
            } else {
              vals[4 * c + 0] = bf16x2_to_f16x2(v.x);
              vals[4 * c + 1] = bf16x2_to_f16x2(v.y);
              vals[4 * c + 2] = bf16x2_to_f16x2(v.z);
              vals[4 * c + 3] = bf16x2_to_f16x2(v.w);
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(raw_empty + rs));
          const uint32_t stage = a_it;
          const int as = stage % C::NS;
          ok = mbar_wait_warp(smem_u32(s_empty + (as >> 1)), ((stage / C::NS) & 1) ^ 1, abort_flag,
                              p.status);
          if (!ok) break;
          tc_fence_after();
          const uint32_t col = C::ACC_COLS + as * C::A_COLS +
                               (C::NMAT == 2 ? part * (KA / 2) : part * 16);
          tmem_st16(tl + col, vals);
          if (C::NMAT == 2) tmem_st16(tl + col + 16, vals + 16);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(a_full + as));
        }
        ++raw_it;
        a_it += C::A_PER_RAW;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

// ------------------------------------------------------------------ host

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 2-D tiled map: inner extent `inner` elements (contiguous), `outer` rows of
// `row_bytes`, box (box_inner, box_outer).
static bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
                     uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                     CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

// raw weight-tile map over a stack of `rows` weight rows of K elements
static bool weight_map(CUtensorMap* m, int fmt, const void* w, long long rows, int K) {
  if (fmt == MOE_W_Q4G64)
    return make_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, w, K / 8, rows, (uint64_t)K / 2, 32, BMW,
                    CU_TENSOR_MAP_SWIZZLE_128B);
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w, K, rows, (uint64_t)K * 2, 64, BMW,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}

// bf16 -> fp16, 8 values per thread; values that do not round to a finite
// fp16 are reported as MOE_ERR_RANGE (they become +-inf).
__global__ void __launch_bounds__(256) to_f16_kernel(const uint4* __restrict__ in,
                                                     uint4* __restrict__ out, long long n8,
                                                     int* status) {
  pdl_wait();
  pdl_launch();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  bool ok = true;
  if (i < n8) {
    const uint4 v = in[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a = __uint_as_float(w[j] << 16), b = __uint_as_float(w[j] & 0xFFFF0000u);
      ok &= fabsf(a) < 65520.f && fabsf(b) < 65520.f;
      uint32_t d;
      asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(b), "f"(a));
      o[j] = d;
    }
    out[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (!__all_sync(0xffffffffu, ok) && (threadIdx.x & 31) == 0) report_status(status, MOE_ERR_RANGE);
}

template <int FMT, int EPI, bool GATHER, bool ROUTER>
static cudaError_t run(const Params& p, const CUtensorMap& a, long long units_ub, cudaStream_t s) {
  using C = Cfg<FMT, EPI>;
  auto kern = grouped_tc_kernel<FMT, EPI, GATHER, ROUTER>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const long long grid = units_ub < num_sms() ? units_ub : num_sms();
  if (grid <= 0) return cudaSuccess;
  launch_pdl(kern, (unsigned)grid, kThreads, C::SMEM, s, p, a);
  return cudaGetLastError();
}

// the kernels tile d and F by 128 rows; q4 raw stages span 256 elements of K
static bool tc_shape_ok(const moe_experts& ex) {
  if (ex.d % 128 || ex.F % 128) return false;
  if (ex.fmt == MOE_W_Q4G64) return ex.d % 256 == 0 && ex.F % 256 == 0;
  return ex.fmt == MOE_W_BF16;
}

}  // namespace tc

int tc_block_m() { return tc::BN; }

cudaError_t launch_to_f16(const void* x, long long n, void* x16, int* status, cudaStream_t s) {
  const long long n8 = n / 8;
  if (n8 <= 0) return cudaSuccess;
  launch_pdl(tc::to_f16_kernel, (unsigned)((n8 + 255) / 256), 256, 0, s, (const uint4*)x, (uint4*)x16, n8,
                                                                 status);
  return cudaGetLastError();
}

cudaError_t launch_swiglu_tc(const void* x, int T, const uint32_t* row_map, const int32_t* row_off,
                             const int32_t* tile_off, int R, const moe_experts& ex, void* h,
                             void* x16, int* status, cudaStream_t s) {
  using namespace tc;
  if (!tc_shape_ok(ex)) return cudaErrorNotSupported;
  // the expert GEMMs take fp16 operands: x is converted once into x16 [T][d]
  cudaError_t e = launch_to_f16(x, (long long)T * ex.d, x16, status, s);
  if (e != cudaSuccess) return e;
  CUtensorMap ta;
  if (!weight_map(&ta, ex.fmt, ex.w_gu, (long long)ex.E * 2 * ex.F, ex.d)) return cudaErrorInvalidValue;
  Params p{};
  p.row_off = row_off;
  p.tile_off = tile_off;
  p.E = ex.E;
  p.n_mb = ex.F / BMW;
  p.K = ex.d;
  p.rows_per_group = 2 * ex.F;
  p.up_off = ex.F;
  p.G = ex.d / 64;
  p.scales = (const uint16_t*)ex.s_gu;
  p.biases = (const uint16_t*)ex.b_gu;
  p.row_map = row_map;
  p.b_src = x16;
  p.out = h;
  p.out_ld = ex.F;
  p.m_limit = ex.F;
  p.status = status;
  const long long ub = max_tiles(R, ex.E, BN) * p.n_mb;
  if (ex.fmt == MOE_W_Q4G64) return run<MOE_W_Q4G64, EPI_SWIGLU, true, false>(p, ta, ub, s);
  return run<MOE_W_BF16, EPI_SWIGLU, true, false>(p, ta, ub, s);
}

cudaError_t launch_down_tc(const void* h, const int32_t* row_off, const int32_t* tile_off, int R,
                           const moe_experts& ex, void* ys, int* status, cudaStream_t s) {
  using namespace tc;
  if (!tc_shape_ok(ex)) return cudaErrorNotSupported;
  CUtensorMap ta;
  if (!weight_map(&ta, ex.fmt, ex.w_dn, (long long)ex.E * ex.d, ex.F)) return cudaErrorInvalidValue;
  Params p{};
  p.row_off = row_off;
  p.tile_off = tile_off;
  p.E = ex.E;
  p.n_mb = ex.d / BMW;
  p.K = ex.F;
  p.rows_per_group = ex.d;
  p.up_off = 0;
  p.G = ex.F / 64;
  p.scales = (const uint16_t*)ex.s_dn;
  p.biases = (const uint16_t*)ex.b_dn;
  p.b_src = h;
  p.out = ys;
  p.out_ld = ex.d;
  p.m_limit = ex.d;
  p.status = status;
  const long long ub = max_tiles(R, ex.E, BN) * p.n_mb;
  if (ex.fmt == MOE_W_Q4G64) return run<MOE_W_Q4G64, EPI_STORE_F32, false, false>(p, ta, ub, s);
  return run<MOE_W_BF16, EPI_STORE_F32, false, false>(p, ta, ub, s);
}

cudaError_t launch_router_logits_tc(const void* x, const void* w_router, const float* bias, int T,
                                    int d, int E, float* logits, int* status, cudaStream_t s) {
  using namespace tc;
  // few tokens: the weight-streaming kernel is faster than a 128-row tile
  if (T < 256 || d % 128 != 0) return cudaErrorNotSupported;
  CUtensorMap ta;
  if (!weight_map(&ta, MOE_W_BF16, w_router, E, d)) return cudaErrorInvalidValue;
  Params p{};
  p.E = 1;
  p.n_rows = T;
  p.n_mb = (E + BMW - 1) / BMW;
  p.K = d;
  p.out = logits;
  p.out_ld = E;
  p.m_limit = E;
  p.bias = bias;
  p.b_src = x;
  p.status = status;
  const long long ub = (long long)((T + BN - 1) / BN) * p.n_mb;
  return run<MOE_W_BF16, EPI_STORE_F32, false, true>(p, ta, ub, s);
}

}  // namespace moe
