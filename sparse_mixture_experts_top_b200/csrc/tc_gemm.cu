// Tensor-core grouped GEMMs for the prefill regime (tcgen05 / TMEM / TMA).
//
// DS4Server issue #112, "Kernel contract": work is split into tiles that own
// sorted rows of one expert, found from per-expert tile and row prefix tables
// by binary search; gate|up takes the token rows of each sorted row (gathered
// through row_map) and writes silu(gate) * up; the down projection reads rows
// already sorted by expert. mlx-lm PR #2044, "What": each expert's weights are
// read and dequantised once per tile instead of once per (token, slot).
//
// B200 design (one persistent CTA per SM, 24 warps). A unit of work is one
// token tile x two 128-row weight matrices: gate and up rows of the same
// features (gate|up), or the even and odd rows of a 256-row block (down).
//   * swap-AB: the MMA's M = 128 weight rows, N = the tile's token rows
//     (<= 128, rounded up to 16 per tile), so few rows cost few tensor cycles;
//   * warp 0: TMA of the raw weight tiles (q4 words or bf16, 128-byte rows)
//     of both matrices, and cp.async of the q4 scales and biases;
//   * warp 2: one TMA per k-block of the tile's token rows, from a row-sorted
//     fp16 copy (x gathered through row_map, or h),
//     with one tensor map per tile height (16, 32, ..., 128 rows);
//   * warps 8..23 (dequant, 8 per matrix): each thread owns one weight row
//     (one TMEM lane) and half of every raw stage, dequantises w = s*q + b
//     to fp16 and writes it into TMEM with tcgen05.st, where the MMA takes it
//     as its A operand -- the dequantised tile never goes back through shared
//     memory. Two warps per row keep the conversion, which is bound by the
//     latency of its integer and fp16 chains, off the critical path;
//   * warps 1 and 3 (MMA): one thread each issues the tcgen05.mma of one
//     matrix (A from TMEM, B from shared memory) into its own fp32
//     accumulator. Two issuers, because at small N one thread cannot issue
//     MMAs as fast as the tensor core completes them;
//   * warps 4..7 (epilogue): tcgen05.ld of both accumulators, SwiGLU to fp16
//     (gate|up) or fp16 ys (down). Tiles of at most
//     64 rows alternate between two accumulator buffers, so the epilogue of
//     one overlaps the MMAs of the next.
// The expert GEMMs multiply fp16 operands (x converted once from bf16,
// weights dequantised to fp16, h stored in fp16): 11-bit operands keep the
// rounding of the dequantised weights and of h 8x below bf16's; values
// outside the fp16 range are reported as MOE_ERR_RANGE. The router logits
// have their own kernel below (router_tc_kernel): no dequantisation, both
// operands staged by TMA, kept in bf16, whose products are exact in fp32.
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

constexpr int BN = 128;        // token rows per tile (the sort tables' BM; MMA N at most)
constexpr int BMW = 128;       // weight rows per matrix (MMA M)
constexpr int KA = 64;         // K elements per k-block (one q4 group)
constexpr int NS = 4;          // k-block stages of A in TMEM, released in pairs
constexpr int NB = 6;          // token-row (B) stages in shared memory
// Release barriers: k-blocks 2P and 2P + 1 (pair P, counted over the CTA's
// whole k-block sequence) are released on barrier P % NP, its completion
// P / NP. A waiter may lag the barrier by less than one phase only: the
// next completion of the same barrier covers k-blocks 2NP later, so a ring
// reused at distance D needs D <= 2 NP (the TMEM stages: NS; the B stages:
// NB). A parity wait on a barrier two phases ahead would never succeed.
constexpr int NP = 4;
constexpr int NBOX = BN / 16;  // token-row tensor maps: tile heights 16, 32, ..., 128
constexpr int kMaxE = 1024;    // tile / row tables cached in shared memory
constexpr int kThreads = 768;   // 24 warps
constexpr int kEpiWarp0 = 4;
constexpr int kDqWarp0 = 8;
constexpr long long kWaitCycles = 2000000000LL;   // ~1 s at the B200's clocks

// EPI_SWIGLU / EPI_GEGLU: gate|up, h = act(gate) * up in fp16, the gate
// activation fixed at compile time (a runtime choice in the unrolled
// epilogue cost the SwiGLU kernel a fifth of its speed); EPI_STORE: the
// down projection stores fp16 ys.
// The _HP forms keep h in the permuted K order of dequant_word_perm (within
// every 8 consecutive features, position p holds feature (0, 4, 1, 5, 2, 6,
// 3, 7)[p]): the gate|up kernel writes it so, and the down kernel then
// dequantises its q4 weights in that order too -- 4 integer operations per
// word instead of 9. The whole-layer call uses them; the stage calls keep h
// in feature order.
enum { EPI_SWIGLU = 0, EPI_STORE = 1, EPI_GEGLU = 2, EPI_SWIGLU_HP = 3, EPI_GEGLU_HP = 4,
       EPI_STORE_HP = 5 };
template <int EPI> struct Epi {
  static constexpr bool glu = EPI != EPI_STORE && EPI != EPI_STORE_HP;
  static constexpr bool geglu = EPI == EPI_GEGLU || EPI == EPI_GEGLU_HP;
  static constexpr bool perm_out = EPI == EPI_SWIGLU_HP || EPI == EPI_GEGLU_HP;
  // weights dequantised in the permuted K order (the B rows are x16, or h
  // kept permuted)
  static constexpr bool perm_deq = glu || EPI == EPI_STORE_HP;
};

template <int FMT>
struct Cfg {
  static constexpr bool Q4 = q4_group(FMT) != 0;            // 4-bit, groups of 32, 64 or 128
  static constexpr bool Q8 = FMT == MOE_W_Q8G64;            // 8-bit, groups of 64
  static constexpr bool QUANT = Q4 || Q8;
  static constexpr int GS = Q4 ? q4_group(FMT) : 64;        // K elements per scale and bias
  // K elements per raw stage (its rows are 128 bytes)
  static constexpr int KR = Q4 ? 256 : Q8 ? 128 : 64;
  static constexpr int RAW_MAT = BMW * 128;                 // one matrix: 128 rows x 128 bytes
  static constexpr int RAW_BYTES = 2 * RAW_MAT;
  static constexpr int A_PER_RAW = KR / KA;                 // 4 (q4), 2 (q8) or 1 (bf16)
  static constexpr int NR = 3;                              // raw stages
  // bytes of one row's scales (or biases) in a raw stage: 16, 8 or 4 (q4 g32,
  // g64, g128), 4 (q8)
  static constexpr int SB = QUANT ? (KR / GS) * 2 : 0;
  static constexpr int ACC_COLS = 2 * BN;                   // two accumulators of up to 128 columns
  static constexpr int A_COLS = 2 * (KA / 2);               // TMEM columns of one A stage (2 matrices)
  static constexpr int B_BYTES = BN * 128;
  // scales then biases of a raw stage: [2 arrays][2 matrices][128 rows][SB bytes]
  static constexpr int SCL_BYTES = QUANT ? 2 * 2 * BMW * SB : 0;
  static constexpr int TABLES = 2 * (kMaxE + 1) * 4;
  // (the scale ring starts 128-byte aligned after the tables: its rows of up
  // to 16 bytes are copied and read as 16-byte vectors)
  static constexpr int SMEM =
      1024 + NR * RAW_BYTES + NB * B_BYTES + 1024 + TABLES + 128 + NR * SCL_BYTES;
  static_assert(ACC_COLS + NS * A_COLS <= 512, "accumulators and A stages must fit TMEM");
  static_assert(NS % 2 == 0, "A stages are released in pairs");
  static_assert(NS <= 2 * NP && NB <= 2 * NP, "a ring may not outrun its release barriers");
  static_assert(NB % 2 == 0, "the MMA consumes B stages in pairs");
  static_assert(SMEM <= 232448, "shared memory per CTA");
};

struct Params {
  CUtensorMap tmB[NBOX];     // token rows [rows][K] 16-bit; map i: box 64 x 16(i+1), 128B swizzle
  const int32_t* row_off;
  const int32_t* tile_off;
  int E;               // groups (experts)
  int n_units;         // units (pairs of weight matrices) per token tile
  int unit_rows;       // weight rows from one unit to the next
  int mat_off;         // row offset of matrix 1 from matrix 0 inside a unit
  int row_step;        // rows from one row of a matrix to the next: 1, or 2 when
                       // matrix 0 takes the even and matrix 1 the odd rows
  int K;               // reduction length
  int rows_per_group;  // weight rows per expert in the stacked tensor
  int G;               // q4 groups per weight row (K / 64)
  long long w_rows;    // rows of the stacked weight tensor
  const uint16_t* scales;
  const uint16_t* biases;
  void* out;
  int out_ld;          // elements per output row
  int* status;
  long long wait_limit;  // SM cycles a wait for work may take (moe_set_wait_cycles)
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

// try_wait with a suspend-time hint: a thread whose phase is not complete
// sleeps until it completes or about `ns` nanoseconds pass, instead of
// spinning and taking issue slots from the warps that do the work
__device__ __forceinline__ bool mbar_try_sleep(uint32_t bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase of `parity` to complete: at most `limit` SM
// cycles. Returns false when the kernel is aborting (another role timed out;
// ignored when !honor_abort) or this wait ran out. Waits for work use the
// launch's bound (Params::wait_limit); the waits for copies and MMAs still in
// flight before the CTA exits keep the full bound, so that nothing lands in
// shared memory or TMEM after the CTA has released it. A bound below ~50 us
// also drops the sleep hint, so the wait notices its deadline promptly.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int* status, bool honor_abort = true,
                                          long long limit = kWaitCycles) {
  if (mbar_try(bar, parity)) return true;
  const long long t0 = clock64();
  const bool sleep = limit >= 100000;
  const uint32_t af = smem_u32(const_cast<const int*>(abort_flag));
  for (;;) {
    if (sleep ? mbar_try_sleep(bar, parity, 20000u) : mbar_try(bar, parity)) return true;
    uint32_t aborting;
    asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(aborting) : "r"(af) : "memory");
    if (honor_abort && aborting) return false;
    if (clock64() - t0 > limit) {
      *abort_flag = 1;
      report_status(status, MOE_ERR_TIMEOUT);
      return false;
    }
  }
}

// Every lane waits; the result is the same in all lanes, so the warp stays
// converged for the .sync.aligned tcgen05 instructions that follow.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity,
                                               volatile int* abort_flag, int* status,
                                               bool honor_abort = true,
                                               long long limit = kWaitCycles) {
  const bool r = mbar_wait(bar, parity, abort_flag, status, honor_abort, limit);
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

// The four MMAs of one 64-deep k-block (K-steps of 16) into one accumulator,
// in a single statement: D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16 (fp16 or
// bf16 operands, fp32 accumulation). A columns advance 8 per K-step, the B
// descriptor's start address 32 bytes (+2 in 16-byte units) inside the
// 128-byte swizzle atom; accumulate unless `first`. The whole warp executes
// it with warp-uniform operands and one elected lane issues: issued from a
// single active lane, a tcgen05.mma is accepted only every ~50 cycles; from
// an elected lane of a converged warp the tensor core is the limit (~24
// cycles at N = 48).
__device__ __forceinline__ void mma_kblock(uint32_t d0, uint32_t a0, uint32_t blo, uint32_t bhi,
                                           uint32_t idesc, uint32_t first) {
  asm volatile(
      "{\n\t.reg .pred pf, pt, e;\n\t.reg .b64 b0, b1, b2, b3;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.eq.b32 pf, %5, 0;\n\t"
      "setp.ne.b32 pt, %4, 0;\n\t"
      "mov.b64 b0, {%2, %3};\n\t"
      "add.u32 %2, %2, 2;\n\tmov.b64 b1, {%2, %3};\n\t"
      "add.u32 %2, %2, 2;\n\tmov.b64 b2, {%2, %3};\n\t"
      "add.u32 %2, %2, 2;\n\tmov.b64 b3, {%2, %3};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], b0, %4, pf;\n\t"
      "add.u32 %1, %1, 8;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], b1, %4, pt;\n\t"
      "add.u32 %1, %1, 8;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], b2, %4, pt;\n\t"
      "add.u32 %1, %1, 8;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], b3, %4, pt;\n\t}\n"
      : "+r"(d0), "+r"(a0), "+r"(blo), "+r"(bhi)
      : "r"(idesc), "r"(first)
      : "memory");
}

// address of barrier i of an array of 8-byte mbarriers at shared address base
__device__ __forceinline__ uint32_t bar_at(uint32_t base, uint32_t i) { return base + 8u * i; }

// D[tmem] (+)= A[smem] * B[smem]^T for one 64-deep k-block (four K-steps of
// 16; both descriptors advance 32 bytes inside the 128-byte swizzle atom);
// accumulate unless `first`. Warp-uniform operands, one elected lane issues.
__device__ __forceinline__ void mma_kblock_ss(uint32_t d, uint32_t alo, uint32_t ahi, uint32_t blo,
                                              uint32_t bhi, uint32_t idesc, uint32_t first) {
  asm volatile(
      "{\n\t.reg .pred pf, pt, e;\n\t.reg .b64 a0, a1, a2, a3, b0, b1, b2, b3;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.eq.b32 pf, %6, 0;\n\t"
      "setp.ne.b32 pt, %5, 0;\n\t"
      "mov.b64 a0, {%1, %2};\n\tmov.b64 b0, {%3, %4};\n\t"
      "add.u32 %1, %1, 2;\n\tadd.u32 %3, %3, 2;\n\t"
      "mov.b64 a1, {%1, %2};\n\tmov.b64 b1, {%3, %4};\n\t"
      "add.u32 %1, %1, 2;\n\tadd.u32 %3, %3, 2;\n\t"
      "mov.b64 a2, {%1, %2};\n\tmov.b64 b2, {%3, %4};\n\t"
      "add.u32 %1, %1, 2;\n\tadd.u32 %3, %3, 2;\n\t"
      "mov.b64 a3, {%1, %2};\n\tmov.b64 b3, {%3, %4};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a0, b0, %5, pf;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a1, b1, %5, pt;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a2, b2, %5, pt;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], a3, b3, %5, pt;\n\t}\n"
      : "+r"(d), "+r"(alo), "+r"(ahi), "+r"(blo), "+r"(bhi)
      : "r"(idesc), "r"(first)
      : "memory");
}

// 16 columns of this warp's 32 lanes from one TMEM address, and the wait
__device__ __forceinline__ void tmem_ld16(uint32_t ta, uint32_t (&a)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]),
        "=r"(a[7]), "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]),
        "=r"(a[14]), "=r"(a[15])
      : "r"(ta)
      : "memory");
}

// tcgen05.commit from one elected lane of a converged warp
__device__ __forceinline__ void mma_commit_warp(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}\n" ::"r"(bar)
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

// 16 columns of this warp's 32 lanes from each of two TMEM addresses, and the
// wait for them, in one statement: the destination registers of tcgen05.ld
// are written asynchronously until tcgen05.wait::ld, so the load and its wait
// must not be separated where the compiler could spill or move them.
__device__ __forceinline__ void tmem_ld16x2(uint32_t ta, uint32_t tb, uint32_t (&a)[16],
                                            uint32_t (&b)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%32];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%33];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]),
        "=r"(a[7]), "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]),
        "=r"(a[14]), "=r"(a[15]), "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3]), "=r"(b[4]),
        "=r"(b[5]), "=r"(b[6]), "=r"(b[7]), "=r"(b[8]), "=r"(b[9]), "=r"(b[10]), "=r"(b[11]),
        "=r"(b[12]), "=r"(b[13]), "=r"(b[14]), "=r"(b[15])
      : "r"(ta), "r"(tb)
      : "memory");
}
// 16 (or 2 x 16) columns of this warp's 32 lanes stored and waited for in one
// statement, so no source register is reused while the store is in flight.
__device__ __forceinline__ void tmem_st16_sync(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st32_sync(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
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

// The same for a permuted K order: out[c] holds elements (c, c + 4) of the
// word. A nibble at bits 0..3 of a 16-bit half becomes the mantissa of
// fp16 1024.0 (0x6400 | q = 1024 + q); one at bits 4..7 becomes mantissa
// bits 4..7 of fp16 64.0, whose last place is 1/16 (0x5400 | 16q = 64 + q).
// Pairs (e0,e4) and (e1,e5) are one AND-OR each. For (e2,e6) and (e3,e7) a
// byte permute puts bytes 1 and 3 of the word (e3:e2, e7:e6) under the
// exponent of 1024, giving 1024 + 16 e3 + e2 (and e7, e6); one AND-OR of that
// gives 64 + e3, and e2 = (1024 + 16 e3 + e2) - 16 (64 + e3) exactly. The
// magic numbers are subtracted exactly and one fused multiply-add applies
// the scale and bias, rounding once: 4 integer and 8 fp16 operations per
// word. The other operand must use the same order: within every 8
// consecutive K elements, position p holds element (0, 4, 1, 5, 2, 6, 3, 7)[p].
__device__ __forceinline__ void dequant_word_perm(uint32_t w, uint32_t s2, uint32_t b2,
                                                  uint32_t* out) {
  const uint32_t c1024 = 0x64006400u, c64 = 0x54005400u, m16 = 0xCC00CC00u;   // -16.0
  const uint32_t hi = __byte_perm(w, 0x64646464u, 0x4341);                   // 1024 + 16 e3 + e2
  const uint32_t d = (hi & 0x00F000F0u) | c64;                               // 64 + e3
  out[0] = f16x2_fma(f16x2_sub((w & 0x000F000Fu) | c1024, c1024), s2, b2);    // e0, e4
  out[1] = f16x2_fma(f16x2_sub((w & 0x00F000F0u) | c64, c64), s2, b2);        // e1, e5
  out[2] = f16x2_fma(f16x2_fma(d, m16, hi), s2, b2);                          // e2, e6
  out[3] = f16x2_fma(f16x2_sub(d, c64), s2, b2);                              // e3, e7
}

// 4 bytes of one word (element j in byte j) -> 2 fp16 pairs of s * q + b in K
// order: a byte permute puts each byte under the exponent of fp16 1024.0
// (0x64qq = 1024 + q, exact for q <= 255), the magic is subtracted exactly and
// one fused multiply-add applies scale and bias, rounding once.
__device__ __forceinline__ void dequant_word_q8(uint32_t w, uint32_t s2, uint32_t b2,
                                                uint32_t* out) {
  const uint32_t c1024 = 0x64006400u;
  out[0] = f16x2_fma(f16x2_sub(__byte_perm(w, 0x64646464u, 0x4140), c1024), s2, b2);  // q0, q1
  out[1] = f16x2_fma(f16x2_sub(__byte_perm(w, 0x64646464u, 0x4342), c1024), s2, b2);  // q2, q3
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// ------------------------------------------------------------------ tiles

// Work item u -> (unit within the tile, first sorted row r0, valid rows nv,
// expert e), with the prefix tables read from their shared-memory copies.
__device__ __forceinline__ void decode_unit(const Params& p, const int* s_toff, const int* s_roff,
                                            int u, int& unit, int& r0, int& nv, int& e) {
  const int tau = u / p.n_units;
  unit = u - tau * p.n_units;
  int lo = 0, hi = p.E - 1;      // largest e with tile_off[e] <= tau
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_toff[mid] <= tau) lo = mid; else hi = mid - 1;
  }
  e = lo;
  r0 = s_roff[e] + (tau - s_toff[e]) * BN;
  nv = min(BN, s_roff[e + 1] - r0);
}

__device__ __forceinline__ int total_units(const Params& p, const int* s_toff) {
  return s_toff[p.E] * p.n_units;
}

// MMA N of a tile: its rows rounded up to 16
__device__ __forceinline__ int mma_n(int nv) { return max(16, (nv + 15) & ~15); }

// ------------------------------------------------------------------ kernel

template <int FMT, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_tc_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tmA) {
  using C = Cfg<FMT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  const uint32_t raw_base = smem_u32(smem);
  const uint32_t b_base = raw_base + C::NR * C::RAW_BYTES;
  uint8_t* bar_area = smem + C::NR * C::RAW_BYTES + NB * C::B_BYTES;
  uint64_t* raw_full = reinterpret_cast<uint64_t*>(bar_area);   // [NR]
  uint64_t* raw_empty = raw_full + C::NR;                        // [NR]
  uint64_t* a_full = raw_empty + C::NR;                          // [2 matrices][NS]
  uint64_t* b_full = a_full + 2 * NS;                            // [NB / 2] B stage pairs
  uint64_t* s_empty = b_full + NB / 2;                           // [NP] k-block pair releases
  uint64_t* acc_full = s_empty + NP;                             // [2] accumulator buffers
  uint64_t* acc_empty = acc_full + 2;                            // [2]
  uint64_t* drain = acc_empty + 2;                               // [2] one per issuer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // shared-memory addresses of the barrier arrays
  const uint32_t raw_full_s = smem_u32(raw_full);
  const uint32_t raw_empty_s = smem_u32(raw_empty);
  const uint32_t b_full_s = smem_u32(b_full);
  const uint32_t s_empty_s = smem_u32(s_empty);
  const uint32_t acc_full_s = smem_u32(acc_full);
  const uint32_t acc_empty_s = smem_u32(acc_empty);
  const uint32_t drain_s = smem_u32(drain);
  // one scratch word per warp (see the dequant role)
  const uint32_t sink = smem_u32(bar_area + 512);
  int* s_toff = reinterpret_cast<int*>(bar_area + 1024);
  int* s_roff = s_toff + kMaxE + 1;
  // scale ring: raw stage rs holds scales [2][128][SB bytes] then biases,
  // 128-byte aligned
  const uint32_t scl_base = (smem_u32(s_roff + kMaxE + 1) + 127u) & ~127u;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NR; ++i) {
      // quantised: the TMA arrive + the 32 lanes' cp.async arrivals for the scales
      mbar_init(bar_at(raw_full_s, i), C::QUANT ? 33 : 1);
      mbar_init(bar_at(raw_empty_s, i), 16);   // the 16 dequant warps
    }
    // one barrier per A stage pair of a matrix: quantised, each stage of the
    // pair is written by the 4 warps of one half (8 arrivals); bf16, each
    // stage by the 8 warps of both halves (16 arrivals)
    for (int i = 0; i < 2 * NS; ++i) mbar_init(smem_u32(a_full + i), C::QUANT ? 8 : 16);
    for (int i = 0; i < NB / 2; ++i) mbar_init(bar_at(b_full_s, i), 1);
    for (int i = 0; i < NP; ++i) mbar_init(bar_at(s_empty_s, i), 2);   // both issuers
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_at(acc_full_s, i), 2);    // both issuers
      mbar_init(bar_at(acc_empty_s, i), 4);   // the 4 epilogue warps
      mbar_init(bar_at(drain_s, i), 1);
    }
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
  for (int i = threadIdx.x; i <= p.E; i += blockDim.x) {
    s_toff[i] = __ldg(p.tile_off + i);
    s_roff[i] = __ldg(p.row_off + i);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int total = total_units(p, s_toff);
  const int nkr = p.K / C::KR;           // raw stages per unit
  const int nka = p.K / KA;              // k-blocks per unit (even: K % 128 == 0)

  if (warp == 0) {
    // ------------------------------------------------------------ raw weights (TMA)
    uint32_t raw_it = 0, rs = 0, rph = 0;      // stages issued; ring slot and its phase
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
      int unit, r0, nv, e;
      decode_unit(p, s_toff, s_roff, u, unit, r0, nv, e);
      const long long wrow0 = (long long)e * p.rows_per_group + (long long)unit * p.unit_rows;
      const long long wrow1 = wrow0 + p.mat_off;
      for (int kr = 0; kr < nkr && ok; ++kr) {
        ok = mbar_wait_warp(bar_at(raw_empty_s, rs), rph ^ 1, abort_flag, p.status, true,
                            p.wait_limit);
        if (!ok) break;
        if (C::QUANT) {
          // the stage's scales and biases (KR / GS groups of each weight
          // row), SB bytes per row and array, copied by the 32 lanes; each
          // lane's arrival fires when its copies have landed. Rows past the
          // end of the stacked tensor (never stored) read the last row instead.
          const uint32_t sdst = scl_base + rs * C::SCL_BYTES;
#pragma unroll
          for (int mat = 0; mat < 2; ++mat)
#pragma unroll
            for (int j = 0; j < BMW / 32; ++j) {
              const int m = lane + 32 * j;
              long long grow = (mat ? wrow1 : wrow0) + (long long)m * p.row_step;
              if (grow >= p.w_rows) grow = p.w_rows - 1;
              const uint32_t o = (uint32_t)((mat * BMW + m) * C::SB);
              const long long g0 = grow * p.G + (long long)(C::KR / C::GS) * kr;
              asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(sdst + o),
                           "l"(p.scales + g0), "n"(C::SB)
                           : "memory");
              asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(
                               sdst + C::SCL_BYTES / 2 + o),
                           "l"(p.biases + g0), "n"(C::SB)
                           : "memory");
            }
          asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(
                           bar_at(raw_full_s, rs))
                       : "memory");
        }
        if (lane == 0) {
          // rows past the end of the tensor are filled with zeros by the TMA
          const uint32_t dst = raw_base + rs * C::RAW_BYTES;
          const uint32_t bar = bar_at(raw_full_s, rs);
          const int x = kr * (C::Q4 ? C::KR / 8 : C::Q8 ? C::KR / 4 : C::KR);
          mbar_arrive_tx(bar, C::RAW_BYTES);
          tma_load_2d(dst, &tmA, x, (int)wrow0, bar);
          tma_load_2d(dst + C::RAW_MAT, &tmA, x, (int)wrow1, bar);
        }
        ++raw_it;
        if (++rs == (uint32_t)C::NR) { rs = 0; rph ^= 1; }
      }
    }
    // copies in flight: wait (bounded, also when aborting) for the last
    // phase issued on every stage before the CTA may exit
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (lane == 0) {
      for (uint32_t i = 0; i < (uint32_t)C::NR && i < raw_it; ++i) {
        const uint32_t last = raw_it - 1 - i;
        mbar_wait(bar_at(raw_full_s, last % C::NR), (last / C::NR) & 1, abort_flag, p.status, false);
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------ token rows (TMA)
    // One copy per k-block: rows r0 .. r0 + n - 1 (n = the tile's MMA N) of
    // the row-sorted 16-bit operand, 64 elements (128 bytes) each, landing in
    // the 128B-swizzled K-major layout the MMA reads. Rows past the tile
    // belong to the next tile (their columns are never stored) or lie past
    // the end (zero fill). k-blocks go two at a time (one barrier for the
    // pair); B stages j, j + 1 are reused by k-blocks j + NB, j + NB + 1 once
    // their k-block pair has been released by both issuers.
    if (lane == 0) {
      uint32_t j = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
        int unit, r0, nv, e;
        decode_unit(p, s_toff, s_roff, u, unit, r0, nv, e);
        const int n = mma_n(nv);
        const CUtensorMap* tm = &p.tmB[n / 16 - 1];
        for (int kb = 0; kb < nka && ok; kb += 2) {
          const int bs = j % NB;
          if (j >= (uint32_t)NB) {
            const uint32_t pr = (j - NB) >> 1;
            ok = mbar_wait(bar_at(s_empty_s, pr % NP), (pr / NP) & 1, abort_flag, p.status, true, p.wait_limit);
            if (!ok) break;
          }
          const uint32_t bar = bar_at(b_full_s, bs / 2);
          mbar_arrive_tx(bar, (uint32_t)n * 256u);
          tma_load_2d(b_base + bs * C::B_BYTES, tm, kb * KA, r0, bar);
          tma_load_2d(b_base + (bs + 1) * C::B_BYTES, tm, (kb + 1) * KA, r0, bar);
          j += 2;
        }
      }
      for (uint32_t i = 0; i < (uint32_t)NB && i < j; i += 2) {
        const uint32_t last = (j - 2 - i) / 2;      // pair index
        mbar_wait(bar_at(b_full_s, last % (NB / 2)), (last / (NB / 2)) & 1, abort_flag, p.status,
                  false);
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp == 3) {
    // ------------------------------------------------------------ MMA issuers
    // warp 1 issues matrix 0, warp 3 matrix 1, each into its own
    // accumulator; the whole warp runs the loop (warp-uniform operands) and
    // one elected lane issues
    const int q = warp >> 1;
    const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
    uint32_t ss = 0, sph = 0, bs = 0, bph = 0;        // A and B stage slots and phases
    uint32_t kg = 0;                                  // k-blocks issued so far
    uint32_t nb = 0, uses0 = 0, uses1 = 0;            // accumulator buffers
    bool ok = true;
    // descriptor of B stage 0 (low word: start address / 16 and the
    // leading offset; high word: stride offset, version, swizzle)
    const uint64_t d0 = desc_sw128(b_base);
    const uint32_t blo0 = (uint32_t)d0, bhi = (uint32_t)(d0 >> 32);
    const uint32_t a_col0 = tm + C::ACC_COLS + q * (KA / 2);
    const uint32_t afull0 = smem_u32(a_full + q * NS);
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
      int unit, r0, nv, e;
      decode_unit(p, s_toff, s_roff, u, unit, r0, nv, e);
      const int n = mma_n(nv);
      const uint32_t idesc = idesc_mma(n, true);
      // tiles of <= 64 rows alternate between the two 128-column buffers
      // (matrix q at +64q); larger ones take both (matrix q at +128q)
      const bool small = n <= 64;
      const uint32_t b = small ? nb : 0u;
      const bool use0 = !small || b == 0, use1 = !small || b == 1;
      // the epilogue has drained the buffers' previous tiles
      if (use0 && uses0 > 0)
        ok = mbar_wait_warp(bar_at(acc_empty_s, 0), (uses0 - 1) & 1, abort_flag, p.status, true, p.wait_limit);
      if (ok && use1 && uses1 > 0)
        ok = mbar_wait_warp(bar_at(acc_empty_s, 1), (uses1 - 1) & 1, abort_flag, p.status, true, p.wait_limit);
      if (!ok) break;
      tc_fence_after();
      const uint32_t dcol = tm + (small ? b * 128u + q * 64u : q * 128u);
      // k-blocks two at a time (a unit has an even number of them; NS and
      // NB are even, so both stages of a pair share their phases): two
      // waits, eight MMAs and one release per pair. The pair's two A stages
      // complete one barrier; both B stages share another.
      for (int kb = 0; kb < nka && ok; kb += 2) {
        ok = mbar_wait_warp(afull0 + (ss >> 1) * 8, sph, abort_flag, p.status, true, p.wait_limit) &&
             mbar_wait_warp(bar_at(b_full_s, bs / 2), bph, abort_flag, p.status, true, p.wait_limit);
        if (!ok) break;
        tc_fence_after();
        const uint32_t acol = a_col0 + ss * (uint32_t)C::A_COLS;
        const uint32_t blo = blo0 + bs * (uint32_t)(C::B_BYTES >> 4);
        mma_kblock(dcol, acol, blo, bhi, idesc, kb == 0);
        mma_kblock(dcol, acol + C::A_COLS, blo + (C::B_BYTES >> 4), bhi, idesc, 0);
        mma_commit_warp(bar_at(s_empty_s, (kg >> 1) % NP));   // release k-block pair kg / 2
        kg += 2;
        if ((ss += 2) == (uint32_t)NS) { ss = 0; sph ^= 1; }
        if ((bs += 2) == (uint32_t)NB) { bs = 0; bph ^= 1; }
      }
      if (!ok) break;
      if (use0) { mma_commit_warp(bar_at(acc_full_s, 0)); ++uses0; }
      if (use1) { mma_commit_warp(bar_at(acc_full_s, 1)); ++uses1; }
      if (small) nb ^= 1u;
    }
    // all MMAs issued by this warp complete before TMEM is released
    mma_commit_warp(bar_at(drain_s, q));
    mbar_wait_warp(bar_at(drain_s, q), 0, abort_flag, p.status, false);
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
    // ------------------------------------------------------------ epilogue
    const int qd = warp & 3;
    const int m = qd * 32 + lane;                     // weight row of this thread
    const uint32_t tl = tmem + ((uint32_t)(qd * 32) << 16);
    uint32_t nb = 0, uses0 = 0, uses1 = 0;
    // largest fp16 magnitude bits stored: 0x7C00 and above is inf or NaN,
    // i.e. a value that did not round to a finite fp16
    uint32_t hmax = 0;
    for (int u = blockIdx.x; u < total; u += gridDim.x) {
      int unit, r0, nv, e;
      decode_unit(p, s_toff, s_roff, u, unit, r0, nv, e);
      const bool small = mma_n(nv) <= 64;
      const uint32_t b = small ? nb : 0u;
      const bool use0 = !small || b == 0, use1 = !small || b == 1;
      if (use0 && !mbar_wait_warp(bar_at(acc_full_s, 0), uses0 & 1, abort_flag, p.status, true, p.wait_limit)) break;
      if (use1 && !mbar_wait_warp(bar_at(acc_full_s, 1), uses1 & 1, abort_flag, p.status, true, p.wait_limit)) break;
      tc_fence_after();
      const uint32_t c0 = tl + (small ? b * 128u : 0u);         // matrix 0
      const uint32_t c1 = tl + (small ? b * 128u + 64u : 128u);  // matrix 1
      // 16 columns of both accumulators at a time
      if (Epi<EPI>::glu) {
        constexpr int kAct = Epi<EPI>::geglu ? MOE_ACT_GEGLU_TANH : MOE_ACT_SWIGLU;
        int orow = unit * p.unit_rows + m;                // feature of this thread
        // feature 8g + i at position 8g + 2 (i % 4) + i / 4 (unit_rows % 8 == 0)
        if (Epi<EPI>::perm_out) orow = (orow & ~7) | ((orow & 3) << 1) | ((orow >> 2) & 1);
        __half* hp = reinterpret_cast<__half*>(p.out) + (size_t)r0 * p.out_ld + orow;
        for (int n0 = 0; n0 < nv; n0 += 16) {
          uint32_t a0[16], a1[16];
          tmem_ld16x2(c0 + n0, c1 + n0, a0, a1);
          const int lim = nv - n0;        // columns of this chunk that are rows of the tile
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const __half v =
                __float2half_rn(glu(kAct, __uint_as_float(a0[j]), __uint_as_float(a1[j])));
            if (j < lim) {
              hmax = max(hmax, (uint32_t)__half_as_ushort(v) & 0x7FFFu);
              hp[(size_t)(n0 + j) * p.out_ld] = v;
            }
          }
        }
      } else {
        // the down projection's units are 256 whole rows of d (d % 256 ==
        // 0): matrix 0 holds the even, matrix 1 the odd output features,
        // so this thread's two features are adjacent and each token's
        // pair goes out as one 4-byte store (a warp writes 128 contiguous
        // bytes of a ys row)
        const int of = unit * p.unit_rows + 2 * m;
        uint32_t* op = reinterpret_cast<uint32_t*>(reinterpret_cast<__half*>(p.out) +
                                                   (size_t)r0 * p.out_ld + of);
        const size_t ld2 = (size_t)p.out_ld / 2;
        for (int n0 = 0; n0 < nv; n0 += 16) {
          uint32_t a0[16], a1[16];
          tmem_ld16x2(c0 + n0, c1 + n0, a0, a1);
          const int lim = nv - n0;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const uint32_t v = f16x2_pack(__uint_as_float(a0[j]), __uint_as_float(a1[j]));
            if (j < lim) {
              hmax = __vmaxu2(hmax, v & 0x7FFF7FFFu);    // both halves' magnitudes
              op[(size_t)(n0 + j) * ld2] = v;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (use0) mbar_arrive(bar_at(acc_empty_s, 0));
        if (use1) mbar_arrive(bar_at(acc_empty_s, 1));
      }
      if (use0) ++uses0;
      if (use1) ++uses1;
      if (small) nb ^= 1u;
    }
    // (down: the two 16-bit halves hold separate maxima)
    const uint32_t hm = max(hmax & 0xFFFFu, hmax >> 16);
    if (!__all_sync(0xffffffffu, hm < 0x7C00u) && lane == 0) report_status(p.status, MOE_ERR_RANGE);
  } else if (warp >= kDqWarp0) {
    // ------------------------------------------------------------ dequant
    // 16 warps: (matrix q, lane quadrant qd, half hf). q4: half hf converts
    // k-blocks hf and 2 + hf of every raw stage (chunks 2hf, 2hf + 1 and
    // 4 + 2hf, 5 + 2hf of the row), so both halves fill a k-block pair
    // together and the MMAs of one pair overlap the conversion of the next;
    // q8: half hf converts k-block hf (chunks 4hf .. 4hf + 3); bf16: half hf
    // converts K elements 32hf .. 32hf + 31 of the raw stage's single A stage.
    const int dw = warp - kDqWarp0;                   // 0..15
    const int q = (dw >> 2) & 1;                      // matrix
    const int hf = dw >> 3;                           // half of the raw stage
    const int qd = warp & 3;                          // TMEM lane quadrant
    const int m = qd * 32 + lane;                     // weight row of this thread
    const uint32_t tl = tmem + ((uint32_t)(qd * 32) << 16);
    const uint32_t afull = smem_u32(a_full + q * NS);
    constexpr int NST = C::Q4 ? 2 : 1;                // A stages per raw stage of this warp
    uint32_t rs = 0, rph = 0, a_it = 0;         // raw ring slot and its phase
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
      for (int kr = 0; kr < nkr && ok; ++kr) {
        ok = mbar_wait_warp(bar_at(raw_full_s, rs), rph, abort_flag, p.status, true, p.wait_limit);
        if (!ok) break;
        // my half row: 4 chunks of 16 B in the 128-byte swizzle
        const uint32_t rowa = raw_base + rs * C::RAW_BYTES + q * C::RAW_MAT + m * 128;
        const int sw = m & 7;
        uint4 wv[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int chunk = C::Q4 ? 2 * hf + c + (c & 2) : 4 * hf + c;
          wv[c] = lds128(rowa + (((uint32_t)chunk ^ (uint32_t)sw) << 4));
        }
        // this row's scales and biases for the warp's A stage j, as bf16 in
        // the low half (and, groups of 32, the second group of the k-block
        // in the high half)
        uint32_t sg[2] = {0u, 0u}, bg[2] = {0u, 0u};
        if (C::QUANT) {
          const uint32_t so = scl_base + rs * C::SCL_BYTES + (uint32_t)((q * BMW + m) * C::SB);
          const uint32_t bo = so + C::SCL_BYTES / 2;
          if (C::SB == 16) {             // q4 g32: k-block kb has groups 2kb, 2kb + 1
            uint32_t sv[4], bv[4];
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(sv[0]), "=r"(sv[1]), "=r"(sv[2]), "=r"(sv[3]) : "r"(so));
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(bv[0]), "=r"(bv[1]), "=r"(bv[2]), "=r"(bv[3]) : "r"(bo));
            sg[0] = hf ? sv[1] : sv[0];
            sg[1] = hf ? sv[3] : sv[2];
            bg[0] = hf ? bv[1] : bv[0];
            bg[1] = hf ? bv[3] : bv[2];
          } else if (C::SB == 8) {       // q4 g64: group kb
            uint32_t s01, s23, b01, b23;
            asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(s01), "=r"(s23) : "r"(so));
            asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(b01), "=r"(b23) : "r"(bo));
            sg[0] = hf ? (s01 >> 16) : (s01 & 0xFFFFu);
            sg[1] = hf ? (s23 >> 16) : (s23 & 0xFFFFu);
            bg[0] = hf ? (b01 >> 16) : (b01 & 0xFFFFu);
            bg[1] = hf ? (b23 >> 16) : (b23 & 0xFFFFu);
          } else {                       // 2 groups: q4 g128 (kb / 2), q8 (kb)
            uint32_t s01, b01;
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(s01) : "r"(so));
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(b01) : "r"(bo));
            if (C::Q4) {
              sg[0] = s01 & 0xFFFFu, sg[1] = s01 >> 16;
              bg[0] = b01 & 0xFFFFu, bg[1] = b01 >> 16;
            } else {
              sg[0] = hf ? (s01 >> 16) : (s01 & 0xFFFFu);
              bg[0] = hf ? (b01 >> 16) : (b01 & 0xFFFFu);
            }
          }
        }
        // A shared-memory load has read its data only once an instruction has
        // consumed its destination registers; until then the next TMA into
        // this stage can overwrite rows the load has not read yet (seen on
        // the first rows the TMA writes). So the loaded words are folded into
        // one value stored to a scratch word before the stage is released.
        // (one register of each vector load: its destination registers are
        // written together, so consuming one waits for the whole load)
        uint32_t fold = sg[0] ^ bg[0];
#pragma unroll
        for (int c = 0; c < 4; ++c) fold ^= wv[c].x;
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(sink + 4u * (uint32_t)warp), "r"(fold)
                     : "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_at(raw_empty_s, rs));
#pragma unroll
        for (int j = 0; j < NST; ++j) {
          uint32_t vals[32];
          if (C::Q4) {
            // my chunks 2j, 2j + 1 hold the 64 elements of k-block hf + 2j of
            // the raw stage; groups of 32: words 0-3 and 4-7 have a group each
            const uint32_t s2 = f16x2_from_bf16(sg[j] & 0xFFFFu);
            const uint32_t b2 = f16x2_from_bf16(bg[j] & 0xFFFFu);
            const uint32_t s2h = C::GS == 32 ? f16x2_from_bf16(sg[j] >> 16) : s2;
            const uint32_t b2h = C::GS == 32 ? f16x2_from_bf16(bg[j] >> 16) : b2;
            const uint4 w0 = wv[2 * j], w1 = wv[2 * j + 1];
            const uint32_t ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              // gate|up reads token rows the gather wrote in permuted order,
              // the _HP down a permuted h
              const uint32_t si = i < 4 ? s2 : s2h, bi = i < 4 ? b2 : b2h;
              if (Epi<EPI>::perm_deq) dequant_word_perm(ws[i], si, bi, vals + 4 * i);
              else dequant_word(ws[i], si, bi, vals + 4 * i);
            }
          } else if (C::Q8) {
            // the 64 bytes of k-block hf, in K order
            const uint32_t s2 = f16x2_from_bf16(sg[0]), b2 = f16x2_from_bf16(bg[0]);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const uint32_t w4[4] = {wv[c].x, wv[c].y, wv[c].z, wv[c].w};
#pragma unroll
              for (int i = 0; i < 4; ++i) dequant_word_q8(w4[i], s2, b2, vals + 8 * c + 2 * i);
            }
          } else {
            // bf16 weights: 32 elements of the k-block; fp16 operands for
            // the experts, bf16 kept as is for the router
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const uint32_t w4[4] = {wv[c].x, wv[c].y, wv[c].z, wv[c].w};
#pragma unroll
              for (int i = 0; i < 4; ++i) vals[4 * c + i] = bf16x2_to_f16x2(w4[i]);
            }
          }
          const uint32_t stage = a_it + (C::Q4 ? hf + 2 * j : C::Q8 ? hf : 0);
          const uint32_t as = stage % NS;
          if (stage >= (uint32_t)NS) {      // the slot's previous k-block is released
            const uint32_t pr = (stage - NS) >> 1;
            ok = mbar_wait_warp(bar_at(s_empty_s, pr % NP), (pr / NP) & 1, abort_flag, p.status, true, p.wait_limit);
            if (!ok) break;
          }
          tc_fence_after();
          const uint32_t col = C::ACC_COLS + as * C::A_COLS + q * (KA / 2) + (C::QUANT ? 0 : hf * 16);
          if (C::QUANT) tmem_st32_sync(tl + col, vals);
          else tmem_st16_sync(tl + col, vals);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(afull + (as >> 1) * 8);
        }
        if (++rs == (uint32_t)C::NR) { rs = 0; rph ^= 1; }
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

// ------------------------------------------------------------------ bf16 gate|up

// gate|up for bf16 weights and bf16 activations: nothing to dequantise, so
// both operands go to the tensor core as loaded (mlx-lm PR #2044, "What":
// the expert's weight tile is read once per token tile; DS4Server issue
// #112, "Kernel contract": h = silu(gate) * up in sorted row order). A unit
// is one token tile x the gate and up rows of 128 features, as in
// grouped_tc_kernel; warp 0 loads each 64-wide k-block of both weight
// matrices and of the tile's token rows (bf16, gathered without conversion)
// by TMA into a ring of SST stages, warp 1 issues the MMAs of both matrices
// (A and B in shared memory) into two accumulators, warps 2..5 apply the GLU.
// The products of bf16 values are exact in fp32, so h is what the fp16
// operand path computes.
constexpr int SST = 4;                          // k-block stages
constexpr int kSThreads = 192;
constexpr int S_A_BYTES = BMW * 128;            // 128 rows x 64 elements, one matrix
constexpr int S_STAGE = 2 * S_A_BYTES + BN * 128;
constexpr int S_SMEM = 1024 + SST * S_STAGE + 256 + 2 * (kMaxE + 1) * 4;
static_assert(S_SMEM <= 232448, "shared memory per CTA");

template <int EPI>
__global__ void __launch_bounds__(kSThreads, 1)
    ss_glu_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tmA) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  const uint32_t st_base = smem_u32(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SST * S_STAGE);   // [SST]
  uint64_t* empty = full + SST;                                         // [SST]
  uint64_t* acc_full = empty + SST;                                     // [2]
  uint64_t* acc_empty = acc_full + 2;                                   // [2]
  uint64_t* drain = acc_empty + 2;                                      // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_toff = reinterpret_cast<int*>(smem + SST * S_STAGE + 256);
  int* s_roff = s_toff + kMaxE + 1;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < SST; ++i) {
      mbar_init(smem_u32(full + i), 1);    // the loader's arrive + the copies' bytes
      mbar_init(smem_u32(empty + i), 1);   // the MMAs' commit
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(acc_full + i), 1);
      mbar_init(smem_u32(acc_empty + i), 4);   // the 4 epilogue warps
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
  }
  if (warp == 1) {
    // two accumulator buffers of 128 columns (gate and up of a tile of up to
    // 64 rows each), or both for a larger tile
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 256;" ::"r"(
                     smem_u32(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  pdl_wait();
  pdl_launch();
  for (int i = threadIdx.x; i <= p.E; i += blockDim.x) {
    s_toff[i] = __ldg(p.tile_off + i);
    s_roff[i] = __ldg(p.row_off + i);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int total = total_units(p, s_toff);
  const int nk = p.K / KA;

  if (warp == 0) {
    // ------------------------------------------------------------ loads (TMA)
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
        int unit, r0, nv, e;
        decode_unit(p, s_toff, s_roff, u, unit, r0, nv, e);
        const int n = mma_n(nv);
        const CUtensorMap* tb = &p.tmB[n / 16 - 1];
        const int wrow0 = (int)((long long)e * p.rows_per_group + (long long)unit * p.unit_rows);
        for (int kb = 0; kb < nk && ok; ++kb, ++it) {
          const uint32_t s = it % SST;
          if (it >= (uint32_t)SST) {
            ok = mbar_wait(smem_u32(empty + s), ((it / SST) - 1) & 1, abort_flag, p.status, true,
                           p.wait_limit);
            if (!ok) break;
          }
          const uint32_t dst = st_base + s * S_STAGE;
          const uint32_t bar = smem_u32(full + s);
          // weight rows past the stacked tensor and token rows past R are
          // zero-filled; token rows past the tile are never stored
          mbar_arrive_tx(bar, (uint32_t)(2 * S_A_BYTES + n * 128));
          tma_load_2d(dst, &tmA, kb * KA, wrow0, bar);
          tma_load_2d(dst + S_A_BYTES, &tmA, kb * KA, wrow0 + p.mat_off, bar);
          tma_load_2d(dst + 2 * S_A_BYTES, tb, kb * KA, r0, bar);
        }
      }
      for (uint32_t i = 0; i < (uint32_t)SST && i < it; ++i) {
        const uint32_t last = it - 1 - i;
        mbar_wait(smem_u32(full + last % SST), (last / SST) & 1, abort_flag, p.status, false);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
    const uint64_t da = desc_sw128(st_base), db = desc_sw128(st_base + 2 * S_A_BYTES);
    const uint32_t alo0 = (uint32_t)da, ahi = (uint32_t)(da >> 32);
    const uint32_t blo0 = (uint32_t)db, bhi = (uint32_t)(db >> 32);
    uint32_t it = 0, nb = 0, uses0 = 0, uses1 = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
      int unit, r0, nv, e;
      decode_unit(p, s_toff, s_roff, u, unit, r0, nv, e);
      const int n = mma_n(nv);
      const uint32_t idesc = idesc_mma(n, false);      // bf16 operands
      const bool small = n <= 64;
      const uint32_t b = small ? nb : 0u;
      const bool use0 = !small || b == 0, use1 = !small || b == 1;
      if (use0 && uses0 > 0)
        ok = mbar_wait_warp(smem_u32(acc_empty + 0), (uses0 - 1) & 1, abort_flag, p.status, true, p.wait_limit);
      if (ok && use1 && uses1 > 0)
        ok = mbar_wait_warp(smem_u32(acc_empty + 1), (uses1 - 1) & 1, abort_flag, p.status, true, p.wait_limit);
      if (!ok) break;
      tc_fence_after();
      const uint32_t d0 = tm + (small ? b * 128u : 0u);           // gate
      const uint32_t d1 = tm + (small ? b * 128u + 64u : 128u);   // up
      for (int kb = 0; kb < nk && ok; ++kb, ++it) {
        const uint32_t s = it % SST;
        ok = mbar_wait_warp(smem_u32(full + s), (it / SST) & 1, abort_flag, p.status, true,
                            p.wait_limit);
        if (!ok) break;
        tc_fence_after();
        const uint32_t off = s * (uint32_t)(S_STAGE >> 4);
        mma_kblock_ss(d0, alo0 + off, ahi, blo0 + off, bhi, idesc, kb == 0);
        mma_kblock_ss(d1, alo0 + off + (S_A_BYTES >> 4), ahi, blo0 + off, bhi, idesc, kb == 0);
        mma_commit_warp(smem_u32(empty + s));
      }
      if (!ok) break;
      if (use0) { mma_commit_warp(smem_u32(acc_full + 0)); ++uses0; }
      if (use1) { mma_commit_warp(smem_u32(acc_full + 1)); ++uses1; }
      if (small) nb ^= 1u;
    }
    mma_commit_warp(smem_u32(drain));
    mbar_wait_warp(smem_u32(drain), 0, abort_flag, p.status, false);
  } else {
    // ------------------------------------------------------------ epilogue
    constexpr int kAct = Epi<EPI>::geglu ? MOE_ACT_GEGLU_TANH : MOE_ACT_SWIGLU;
    const int qd = warp & 3;
    const int m = qd * 32 + lane;                     // feature of the unit
    const uint32_t tl = tmem + ((uint32_t)(qd * 32) << 16);
    uint32_t nb = 0, uses0 = 0, uses1 = 0, hmax = 0;
    for (int u = blockIdx.x; u < total; u += gridDim.x) {
      int unit, r0, nv, e;
      decode_unit(p, s_toff, s_roff, u, unit, r0, nv, e);
      const bool small = mma_n(nv) <= 64;
      const uint32_t b = small ? nb : 0u;
      const bool use0 = !small || b == 0, use1 = !small || b == 1;
      if (use0 && !mbar_wait_warp(smem_u32(acc_full + 0), uses0 & 1, abort_flag, p.status, true, p.wait_limit)) break;
      if (use1 && !mbar_wait_warp(smem_u32(acc_full + 1), uses1 & 1, abort_flag, p.status, true, p.wait_limit)) break;
      tc_fence_after();
      const uint32_t c0 = tl + (small ? b * 128u : 0u);
      const uint32_t c1 = tl + (small ? b * 128u + 64u : 128u);
      __half* hp = reinterpret_cast<__half*>(p.out) + (size_t)r0 * p.out_ld + unit * p.unit_rows + m;
      for (int n0 = 0; n0 < nv; n0 += 16) {
        uint32_t a0[16], a1[16];
        tmem_ld16x2(c0 + n0, c1 + n0, a0, a1);
        const int lim = nv - n0;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const __half v = __float2half_rn(glu(kAct, __uint_as_float(a0[j]), __uint_as_float(a1[j])));
          if (j < lim) {
            hmax = max(hmax, (uint32_t)__half_as_ushort(v) & 0x7FFFu);
            hp[(size_t)(n0 + j) * p.out_ld] = v;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (use0) mbar_arrive(smem_u32(acc_empty + 0));
        if (use1) mbar_arrive(smem_u32(acc_empty + 1));
      }
      if (use0) ++uses0;
      if (use1) ++uses1;
      if (small) nb ^= 1u;
    }
    if (!__all_sync(0xffffffffu, hmax < 0x7C00u) && lane == 0) report_status(p.status, MOE_ERR_RANGE);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 256;" ::"r"(tmem) : "memory");
  }
}

// ------------------------------------------------------------------ router

// Router logits on the tensor cores, both operands staged in shared memory
// by TMA: logits[t][e] = sum_k x[t][k] * W_r[e][k] (+ bias[e]), fp32
// accumulation of exact bf16 (or fp16) products. ("5.5 real sparse MoE
// kernels (Metal)", Scope -- in: router logits, softmax, top-k.)
// A unit is 128 experts (the MMA's M: router weight rows) x one tile of rn
// tokens (its N: x rows); the CTA streams both through a ring of RST stages
// of one 64-wide k-block each. Warp 0 loads, warp 1 issues the MMAs (one
// elected lane), warps 2..5 move the accumulator out: lane = expert, so a
// warp's 32 lanes store 128 contiguous bytes of one token's logits. Two
// accumulator buffers let the epilogue of one unit overlap the MMAs of the
// next. Nothing is converted on the way: unlike the expert GEMMs, whose
// weights must be dequantised, both operands go to the tensor core as loaded.
constexpr int RST = 6;                         // k-block stages
constexpr int kRThreads = 192;                 // 6 warps
constexpr int R_A_BYTES = BMW * 128;           // 128 weight rows x 64 elements
constexpr int R_B_BYTES = BN * 128;            // up to 128 token rows x 64 elements
constexpr int R_STAGE = R_A_BYTES + R_B_BYTES;
constexpr int R_SMEM = 1024 + RST * R_STAGE + 256;
static_assert(R_SMEM <= 232448, "shared memory per CTA");

struct RouterParams {
  int T, E, K;
  int rn;              // token rows per tile (MMA N): 16, 32, 64 or 128
  int n_mblk;          // 128-expert blocks
  int n_units;         // n_mblk x token tiles
  float* logits;       // [T][E]
  const float* bias;   // [E] or null
  int f16;             // x and W_r are fp16 (else bf16)
  int* status;
  long long wait_limit;
};



__global__ void __launch_bounds__(kRThreads, 1)
    router_tc_kernel(const __grid_constant__ RouterParams p, const __grid_constant__ CUtensorMap tmW,
                     const __grid_constant__ CUtensorMap tmX) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  const uint32_t st_base = smem_u32(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + RST * R_STAGE);   // [RST]
  uint64_t* empty = full + RST;                                         // [RST]
  uint64_t* acc_full = empty + RST;                                     // [2]
  uint64_t* acc_empty = acc_full + 2;                                   // [2]
  uint64_t* drain = acc_empty + 2;                                      // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < RST; ++i) {
      mbar_init(smem_u32(full + i), 1);    // the loader's arrive + the copies' bytes
      mbar_init(smem_u32(empty + i), 1);   // the MMAs' commit
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(acc_full + i), 1);
      mbar_init(smem_u32(acc_empty + i), 4);   // the 4 epilogue warps
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmW)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmX)) : "memory");
  }
  if (warp == 1) {
    // two accumulator buffers of up to 128 columns
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 256;" ::"r"(
                     smem_u32(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  pdl_wait();
  pdl_launch();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nk = p.K / KA;

  if (warp == 0) {
    // ------------------------------------------------------------ loads (TMA)
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
        const int mb = u % p.n_mblk, tt = u / p.n_mblk;
        for (int kb = 0; kb < nk && ok; ++kb, ++it) {
          const uint32_t s = it % RST;
          if (it >= (uint32_t)RST) {
            ok = mbar_wait(smem_u32(empty + s), ((it / RST) - 1) & 1, abort_flag, p.status, true,
                           p.wait_limit);
            if (!ok) break;
          }
          const uint32_t dst = st_base + s * R_STAGE;
          const uint32_t bar = smem_u32(full + s);
          // rows past E or T are zero-filled and never stored
          mbar_arrive_tx(bar, (uint32_t)(R_A_BYTES + p.rn * 128));
          tma_load_2d(dst, &tmW, kb * KA, mb * BMW, bar);
          tma_load_2d(dst + R_A_BYTES, &tmX, kb * KA, tt * p.rn, bar);
        }
      }
      // copies in flight complete before the CTA may exit
      for (uint32_t i = 0; i < (uint32_t)RST && i < it; ++i) {
        const uint32_t last = it - 1 - i;
        mbar_wait(smem_u32(full + last % RST), (last / RST) & 1, abort_flag, p.status, false);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
    const uint32_t idesc = idesc_mma(p.rn, p.f16 != 0);
    const uint64_t da = desc_sw128(st_base), db = desc_sw128(st_base + R_A_BYTES);
    const uint32_t alo0 = (uint32_t)da, ahi = (uint32_t)(da >> 32);
    const uint32_t blo0 = (uint32_t)db, bhi = (uint32_t)(db >> 32);
    uint32_t it = 0, n_acc = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x, ++n_acc) {
      const uint32_t buf = n_acc & 1;
      // the epilogue has drained this buffer's previous unit
      if (n_acc >= 2) {
        ok = mbar_wait_warp(smem_u32(acc_empty + buf), ((n_acc >> 1) - 1) & 1, abort_flag,
                            p.status, true, p.wait_limit);
        if (!ok) break;
      }
      tc_fence_after();
      for (int kb = 0; kb < nk && ok; ++kb, ++it) {
        const uint32_t s = it % RST;
        ok = mbar_wait_warp(smem_u32(full + s), (it / RST) & 1, abort_flag, p.status, true,
                            p.wait_limit);
        if (!ok) break;
        tc_fence_after();
        const uint32_t off = s * (uint32_t)(R_STAGE >> 4);
        mma_kblock_ss(tm + buf * 128u, alo0 + off, ahi, blo0 + off, bhi, idesc, kb == 0);
        mma_commit_warp(smem_u32(empty + s));
      }
      if (!ok) break;
      mma_commit_warp(smem_u32(acc_full + buf));
    }
    // all MMAs issued complete before TMEM is released
    mma_commit_warp(smem_u32(drain));
    mbar_wait_warp(smem_u32(drain), 0, abort_flag, p.status, false);
  } else {
    // ------------------------------------------------------------ epilogue
    const int qd = warp & 3;                          // TMEM lane quadrant
    const uint32_t tl = tmem + ((uint32_t)(qd * 32) << 16);
    uint32_t n_acc = 0;
    for (int u = blockIdx.x; u < p.n_units; u += gridDim.x, ++n_acc) {
      const int mb = u % p.n_mblk, tt = u / p.n_mblk;
      const uint32_t buf = n_acc & 1;
      if (!mbar_wait_warp(smem_u32(acc_full + buf), (n_acc >> 1) & 1, abort_flag, p.status, true,
                          p.wait_limit))
        break;
      tc_fence_after();
      const int e = mb * BMW + qd * 32 + lane;
      const bool ok_e = e < p.E;
      const float bv = (ok_e && p.bias) ? __ldg(p.bias + e) : 0.f;
      const int t0 = tt * p.rn;
      float* op = p.logits + (size_t)t0 * p.E + e;
      for (int n0 = 0; n0 < p.rn; n0 += 16) {
        uint32_t a[16];
        tmem_ld16(tl + buf * 128u + (uint32_t)n0, a);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (ok_e && t0 + n0 + j < p.T) op[(size_t)(n0 + j) * p.E] = __uint_as_float(a[j]) + bv;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(acc_empty + buf));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 256;" ::"r"(tmem) : "memory");
  }
}

// Test support: the mbarrier wait of this file made to run out. The barrier
// expects two arrivals and gets one, so the wait must give up after `limit`
// cycles, record MOE_ERR_TIMEOUT and return.
__global__ void wait_selftest_kernel(long long limit, int* status) {
  __shared__ uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 2);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_arrive(smem_u32(&bar));
  __syncwarp();
  mbar_wait_warp(smem_u32(&bar), 0, &abort_flag, status, true, limit);
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
                     CUtensorMapSwizzle sw, uint32_t outer_step = 1) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  // with an outer traversal stride of s the box spans box_outer rows and
  // loads every s-th of them (box_outer / s rows)
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, outer_step};
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
// (16-bit rows are bf16, or fp16 for an fp16 router weight)
// (row_step 2: each load takes every other row, 128 of 256)
static bool weight_map(CUtensorMap* m, int fmt, const void* w, long long rows, int K,
                       bool f16 = false, uint32_t row_step = 1) {
  if (q4_group(fmt) || fmt == MOE_W_Q8G64) {
    // uint32 words: 8 (q4) or 4 (q8) elements each; rows of 128 bytes per box
    const int per = fmt == MOE_W_Q8G64 ? 4 : 8;
    return make_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, w, K / per, rows, (uint64_t)K * 4 / per,
                    32, BMW * row_step, CU_TENSOR_MAP_SWIZZLE_128B, row_step);
  }
  return make_map(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w,
                  K, rows, (uint64_t)K * 2, 64, BMW * row_step, CU_TENSOR_MAP_SWIZZLE_128B,
                  row_step);
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

// bf16 rows gathered into fp16: out[r][:] = fp16(x[row_map[r]][:]), four
// sorted rows per block (8 values per thread per load); values that do not round to a
// finite fp16 are reported as MOE_ERR_RANGE (they become +-inf). PERM stores
// every 8 consecutive elements in the order (0, 4, 1, 5, 2, 6, 3, 7), the K
// order of dequant_word_perm. SRC16 takes 16-bit rows and copies (and
// permutes) their bits as they are: fp16 x for the fp16 operand path, bf16 x
// for the bf16 gate|up kernel.
template <bool PERM, bool SRC16 = false>
__global__ void __launch_bounds__(256) gather_f16_kernel(const uint4* __restrict__ x,
                                                         const uint32_t* __restrict__ row_map,
                                                         long long R, int d8,
                                                         uint4* __restrict__ out, int* status) {
  pdl_wait();
  pdl_launch();
  // 4 rows per block, 64 threads per row, 4 loads in flight per thread
  const long long r = (long long)blockIdx.x * 4 + (threadIdx.x >> 6);
  if (r >= R) return;
  const uint4* src = x + (size_t)__ldg(row_map + r) * d8;
  uint4* dst = out + (size_t)r * d8;
  bool ok = true;
#pragma unroll 4
  for (int c = threadIdx.x & 63; c < d8; c += 64) {
    const uint4 v = __ldg(src + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    if constexpr (SRC16) {
      // halves 2j (low) and 2j+1 (high) of word j; the permuted pairs are
      // (e_j, e_{j+4}) = low or high halves of words j/2 and j/2 + 2
      if (PERM) {
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t a = w[j >> 1], b = w[(j >> 1) + 2];
          o[j] = (j & 1) ? __byte_perm(a, b, 0x7632) : __byte_perm(a, b, 0x5410);
        }
        dst[c] = make_uint4(o[0], o[1], o[2], o[3]);
      } else {
        dst[c] = v;
      }
    } else {
      float f[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        f[2 * j] = __uint_as_float(w[j] << 16);
        f[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
      }
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float lo = PERM ? f[j] : f[2 * j], hi = PERM ? f[j + 4] : f[2 * j + 1];
        ok &= fabsf(lo) < 65520.f && fabsf(hi) < 65520.f;
        uint32_t dd;
        asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(dd) : "f"(hi), "f"(lo));
        o[j] = dd;
      }
      dst[c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  if (!ok) report_status(status, MOE_ERR_RANGE);
}

// The token-row maps of Params: [rows][K] 16-bit elements, one map per tile
// height (16, 32, ..., 128 rows), 64 elements (128 bytes) wide.
static bool token_maps(Params& p, const void* src, bool bf16, long long rows, int K) {
  for (int i = 0; i < NBOX; ++i)
    if (!make_map(&p.tmB[i], bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                  src, (uint64_t)K, (uint64_t)rows, (uint64_t)K * 2, KA, 16 * (i + 1),
                  CU_TENSOR_MAP_SWIZZLE_128B))
      return false;
  return true;
}

template <int FMT, int EPI>
static cudaError_t run(const Params& p, const CUtensorMap& a, long long units_ub, cudaStream_t s) {
  using C = Cfg<FMT>;
  auto kern = grouped_tc_kernel<FMT, EPI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const long long grid = units_ub < num_sms() ? units_ub : num_sms();
  if (grid <= 0) return cudaSuccess;
  launch_pdl(kern, (unsigned)grid, kThreads, C::SMEM, s, p, a);
  return cudaGetLastError();
}

// The kernel for the experts' weight format. The _HP forms are built for
// the q4 formats only (they permute h for the q4 dequant).
template <int EPI>
static cudaError_t run_fmt(int fmt, const Params& p, const CUtensorMap& a, long long ub,
                           cudaStream_t s) {
  constexpr bool hp = EPI == EPI_SWIGLU_HP || EPI == EPI_GEGLU_HP || EPI == EPI_STORE_HP;
  switch (fmt) {
    case MOE_W_Q4G64: return run<MOE_W_Q4G64, EPI>(p, a, ub, s);
    case MOE_W_Q4G32: return run<MOE_W_Q4G32, EPI>(p, a, ub, s);
    case MOE_W_Q4G128: return run<MOE_W_Q4G128, EPI>(p, a, ub, s);
    default: break;
  }
  if constexpr (!hp) {
    if (fmt == MOE_W_Q8G64) return run<MOE_W_Q8G64, EPI>(p, a, ub, s);
    if (fmt == MOE_W_BF16) return run<MOE_W_BF16, EPI>(p, a, ub, s);
  }
  return cudaErrorNotSupported;
}

// Shapes the kernels tile: gate|up units are 128 features (F % 128), down
// units 256 output rows (d % 256); K (d or F) a multiple of 128 for the
// k-block pairs (q8 raw stages), and of 256 for q4 raw stages. Quantised
// weights need their scale and bias arrays 16-byte aligned (the scales of a
// raw stage are copied in pieces of up to 16 bytes).
static bool tc_shape_ok(const moe_experts& ex, int dt) {
  if (ex.d % 256 || ex.F % 128) return false;
  if (dt != MOE_BF16 && dt != MOE_F16) return false;
  if (q4_group(ex.fmt)) return ex.F % 256 == 0;
  if (ex.fmt == MOE_W_Q8G64) return true;
  return ex.fmt == MOE_W_BF16 && dt == MOE_BF16;
}

}  // namespace tc

int tc_block_m() { return tc::BN; }

cudaError_t launch_tc_wait_selftest(long long limit, int* status, cudaStream_t s) {
  tc::wait_selftest_kernel<<<1, 32, 0, s>>>(limit, status);
  return cudaGetLastError();
}

bool tc_shape_supported(int d, int F, int fmt, int dt) {
  moe_experts ex{};
  ex.d = d;
  ex.F = F;
  ex.fmt = (moe_wfmt)fmt;
  return tc::tc_shape_ok(ex, dt);
}

cudaError_t launch_to_f16(const void* x, long long n, void* x16, int* status, cudaStream_t s) {
  const long long n8 = n / 8;
  if (n8 <= 0) return cudaSuccess;
  launch_pdl(tc::to_f16_kernel, (unsigned)((n8 + 255) / 256), 256, 0, s, (const uint4*)x,
             (uint4*)x16, n8, status);
  return cudaGetLastError();
}

cudaError_t launch_swiglu_tc(const void* x, int dt, int T, const uint32_t* row_map,
                             const int32_t* row_off, const int32_t* tile_off, int R,
                             const moe_experts& ex, void* h, void* xs16, int* status,
                             cudaStream_t s, bool h_perm) {
  using namespace tc;
  if (!tc_shape_ok(ex, dt)) return cudaErrorNotSupported;
  (void)T;
  if (R <= 0) return cudaSuccess;
  // the expert GEMMs take fp16 operands in row-sorted order: x gathered
  // through row_map (and converted once, from bf16) into xs16 [R][d]
  // q4 weights are dequantised in a permuted K order, so are the token rows
  const unsigned gblocks = (unsigned)((R + 3) / 4);
  const bool q4 = q4_group(ex.fmt) != 0;
  // bf16 weights with bf16 activations: both operands stay bf16 (the rows are
  // gathered as they are) and go to the tensor core without conversion
  const bool bf16_ss = ex.fmt == MOE_W_BF16 && dt == MOE_BF16;
  if (bf16_ss)
    launch_pdl(gather_f16_kernel<false, true>, gblocks, 256, 0, s, (const uint4*)x, row_map,
               (long long)R, ex.d / 8, (uint4*)xs16, status);
  else if (q4 && dt == MOE_F16)
    launch_pdl(gather_f16_kernel<true, true>, gblocks, 256, 0, s, (const uint4*)x, row_map,
               (long long)R, ex.d / 8, (uint4*)xs16, status);
  else if (q4)
    launch_pdl(gather_f16_kernel<true>, gblocks, 256, 0, s, (const uint4*)x, row_map, (long long)R,
               ex.d / 8, (uint4*)xs16, status);
  else if (dt == MOE_F16)
    launch_pdl(gather_f16_kernel<false, true>, gblocks, 256, 0, s, (const uint4*)x, row_map,
               (long long)R, ex.d / 8, (uint4*)xs16, status);
  else
    launch_pdl(gather_f16_kernel<false>, gblocks, 256, 0, s, (const uint4*)x, row_map, (long long)R,
               ex.d / 8, (uint4*)xs16, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap ta;
  if (!weight_map(&ta, ex.fmt, ex.w_gu, (long long)ex.E * 2 * ex.F, ex.d)) return cudaErrorInvalidValue;
  Params p{};
  if (!token_maps(p, xs16, bf16_ss, R, ex.d)) return cudaErrorInvalidValue;
  p.row_off = row_off;
  p.tile_off = tile_off;
  p.E = ex.E;
  p.n_units = ex.F / BMW;
  p.unit_rows = BMW;
  p.mat_off = ex.F;
  p.row_step = 1;
  p.K = ex.d;
  p.rows_per_group = 2 * ex.F;
  p.G = wq_group(ex.fmt) ? ex.d / wq_group(ex.fmt) : 0;
  p.w_rows = (long long)ex.E * 2 * ex.F;
  p.scales = (const uint16_t*)ex.s_gu;
  p.biases = (const uint16_t*)ex.b_gu;
  p.out = h;
  p.out_ld = ex.F;
  p.status = status;
  p.wait_limit = wait_cycles();
  const long long ub = max_tiles(R, ex.E, BN) * p.n_units;
  const bool geglu = ex.act == MOE_ACT_GEGLU_TANH;
  if (bf16_ss) {
    auto kern = geglu ? ss_glu_kernel<EPI_GEGLU> : ss_glu_kernel<EPI_SWIGLU>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S_SMEM);
    if (e != cudaSuccess) return e;
    const long long grid = ub < num_sms() ? ub : num_sms();
    launch_pdl(kern, (unsigned)grid, kSThreads, S_SMEM, s, p, ta);
    return cudaGetLastError();
  }
  // h in the permuted K order only for q4 weights (the down kernel then
  // dequantises in that order)
  if (q4 && h_perm)
    return geglu ? run_fmt<EPI_GEGLU_HP>(ex.fmt, p, ta, ub, s)
                 : run_fmt<EPI_SWIGLU_HP>(ex.fmt, p, ta, ub, s);
  return geglu ? run_fmt<EPI_GEGLU>(ex.fmt, p, ta, ub, s)
               : run_fmt<EPI_SWIGLU>(ex.fmt, p, ta, ub, s);
}

cudaError_t launch_down_tc(const void* h, const int32_t* row_off, const int32_t* tile_off, int R,
                           const moe_experts& ex, void* ys, int* status, cudaStream_t s,
                           bool h_perm) {
  using namespace tc;
  // h is fp16 whatever the activations' type
  if (!tc_shape_ok(ex, ex.fmt == MOE_W_Q4G64 ? MOE_F16 : MOE_BF16)) return cudaErrorNotSupported;
  if (R <= 0) return cudaSuccess;
  CUtensorMap ta;
  // matrix 0 = the unit's even output rows, matrix 1 = its odd rows
  if (!weight_map(&ta, ex.fmt, ex.w_dn, (long long)ex.E * ex.d, ex.F, false, 2))
    return cudaErrorInvalidValue;
  Params p{};
  if (!token_maps(p, h, false, R, ex.F)) return cudaErrorInvalidValue;
  p.row_off = row_off;
  p.tile_off = tile_off;
  p.E = ex.E;
  p.n_units = ex.d / (2 * BMW);
  p.unit_rows = 2 * BMW;
  p.mat_off = 1;
  p.row_step = 2;
  p.K = ex.F;
  p.rows_per_group = ex.d;
  p.G = wq_group(ex.fmt) ? ex.F / wq_group(ex.fmt) : 0;
  p.w_rows = (long long)ex.E * ex.d;
  p.scales = (const uint16_t*)ex.s_dn;
  p.biases = (const uint16_t*)ex.b_dn;
  p.out = ys;
  p.out_ld = ex.d;
  p.status = status;
  p.wait_limit = wait_cycles();
  const long long ub = max_tiles(R, ex.E, BN) * p.n_units;
  if (q4_group(ex.fmt) && h_perm) return run_fmt<EPI_STORE_HP>(ex.fmt, p, ta, ub, s);
  return run_fmt<EPI_STORE>(ex.fmt, p, ta, ub, s);
}

cudaError_t launch_router_logits_tc(const void* x, int dt, const void* w_router, const float* bias,
                                    int T, int d, int E, float* logits, int* status,
                                    cudaStream_t s) {
  using namespace tc;
  // any token count: 8 us on one B200 from 1 to 2048 tokens at d = 2048,
  // E = 256-512, where the SIMT tile kernel took 170 us from 65 tokens up
  if (T < 1 || d % 128 != 0) return cudaErrorNotSupported;
  if (dt != MOE_BF16 && dt != MOE_F16) return cudaErrorNotSupported;
  const bool f16 = dt == MOE_F16;
  RouterParams p{};
  p.T = T;
  p.E = E;
  p.K = d;
  p.n_mblk = (E + BMW - 1) / BMW;
  // the widest token tile that still gives 3/8 of the SMs a unit: every unit
  // streams its 128 weight rows and its x rows through one SM, and each
  // halving of the tile re-reads the router weight once more from L2 (at
  // T = 2048, E = 512: 128 rows on 64 SMs 13.3 us, 64 rows on 128 SMs 15.4 us)
  int rn = BN;
  while (rn > 16 && (long long)((T + rn - 1) / rn) * p.n_mblk < (3LL * num_sms()) / 8) rn /= 2;
  p.rn = rn;
  p.n_units = ((T + rn - 1) / rn) * p.n_mblk;
  p.logits = logits;
  p.bias = bias;
  p.f16 = f16;
  p.status = status;
  p.wait_limit = wait_cycles();
  CUtensorMap tw, tx;
  const CUtensorMapDataType ty = f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!make_map(&tw, ty, w_router, (uint64_t)d, (uint64_t)E, (uint64_t)d * 2, KA, BMW,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tx, ty, x, (uint64_t)d, (uint64_t)T, (uint64_t)d * 2, KA, (uint32_t)rn,
                CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       R_SMEM);
  if (e != cudaSuccess) return e;
  const int grid = p.n_units < num_sms() ? p.n_units : num_sms();
  launch_pdl(router_tc_kernel, (unsigned)grid, kRThreads, R_SMEM, s, p, tw, tx);
  return cudaGetLastError();
}

}  // namespace moe
