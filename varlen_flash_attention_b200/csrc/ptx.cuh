// Thin inline-PTX wrappers for sm_100a: mbarriers, TMA tensor loads,
// tcgen05 (TMEM allocation, MMA, commit, ld/st, fences) and a few scalar
// helpers.  Every wrapper issues exactly the instruction its name says.
#pragma once

#include <cstdint>
#include <cuda.h>

namespace skptx {

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// Make generic-proxy writes to shared memory visible to the async proxy (TMA store).
// 16-byte shared-memory store (generic proxy).
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- register budget
// Move this warp's register allocation to N (multiple of 8, 24..256).  Every
// warp of a warpgroup executes the same call; an increase waits until other
// warps of the CTA have released enough with a decrease.
template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// ---------------------------------------------------------------- tcgen05
// TMEM allocation: executed by one full warp.
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Warp-collective forms (the *_block and *_elect helpers): the whole warp
// executes the call convergently (so the operands are warp-uniform) and one
// elected lane issues the instruction.

// A whole 128 x N x (16 * KSTEPS) product as one instruction block: one
// elect, then per K step only the descriptor offsets and the MMA, so the
// issuing warp spends about three instructions per MMA (it shares its
// sub-partition with busy softmax warps).  SS form: both operands in shared
// memory, K-major, 128-byte swizzle, 64-column (128 B) sub-tiles kSubOff
// (descriptor units of 16 B) apart; step k adds (k / 4) * kSubOff + (k % 4) * 2
// to both start addresses (32 B per 16 elements inside a sub-tile).
// accumulate == 0: the first step overwrites D.
template <int KSTEPS, uint32_t kSubOff>
__device__ __forceinline__ void mma_ss_block(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  static_assert(KSTEPS == 4 || KSTEPS == 8, "k steps");
#define SKP_SS_STEP(K, ACC)                                                         \
  "add.s64 ta, %1, " #K "; add.s64 tb, %2, " #K ";\n\t"                          \
  "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ta, tb, %3, " ACC ";\n\t"
  if constexpr (KSTEPS == 8) {
    asm volatile(
        "{\n\t.reg .pred e, p;\n\t.reg .b64 ta, tb;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
        SKP_SS_STEP(2, "1") SKP_SS_STEP(4, "1") SKP_SS_STEP(6, "1")
        "add.s64 ta, %1, %5; add.s64 tb, %2, %5;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ta, tb, %3, 1;\n\t"
        "add.s64 ta, %1, %6; add.s64 tb, %2, %6;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ta, tb, %3, 1;\n\t"
        "add.s64 ta, %1, %7; add.s64 tb, %2, %7;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ta, tb, %3, 1;\n\t"
        "add.s64 ta, %1, %8; add.s64 tb, %2, %8;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ta, tb, %3, 1;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "n"(kSubOff), "n"(kSubOff + 2),
        "n"(kSubOff + 4), "n"(kSubOff + 6)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred e, p;\n\t.reg .b64 ta, tb;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
        SKP_SS_STEP(2, "1") SKP_SS_STEP(4, "1") SKP_SS_STEP(6, "1") "}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
  }
#undef SKP_SS_STEP
}

// TS form: A (M x K, K-major) in tensor memory at column a_tmem, 16-bit
// elements packed two per 32-bit column (element k of a row in column k / 2,
// low half for even k), so 8 columns per 16 elements of K; B (K x N,
// MN-major, 128-byte swizzle) in shared
// memory, step k adds k * kBStep (descriptor units) to its start address.
// Steps past ksteps (1..8) are not issued.
template <uint32_t kBStep>
__device__ __forceinline__ void mma_ts_block(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate, int ksteps) {
  asm volatile(
      "{\n\t.reg .pred e, p, q, e_q;\n\t.reg .b64 tb;\n\t.reg .b32 ra;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
      "setp.gt.s32 q, %5, 1; and.pred e_q, e, q;\n\t"
      "add.s32 ra, %1, 8; add.s64 tb, %2, %6;\n\t"
      "@e_q tcgen05.mma.cta_group::1.kind::f16 [%0], [ra], tb, %3, 1;\n\t"
      "setp.gt.s32 q, %5, 2; and.pred e_q, e, q;\n\t"
      "add.s32 ra, %1, 16; add.s64 tb, %2, %7;\n\t"
      "@e_q tcgen05.mma.cta_group::1.kind::f16 [%0], [ra], tb, %3, 1;\n\t"
      "setp.gt.s32 q, %5, 3; and.pred e_q, e, q;\n\t"
      "add.s32 ra, %1, 24; add.s64 tb, %2, %8;\n\t"
      "@e_q tcgen05.mma.cta_group::1.kind::f16 [%0], [ra], tb, %3, 1;\n\t"
      "setp.gt.s32 q, %5, 4; and.pred e_q, e, q;\n\t"
      "add.s32 ra, %1, 32; add.s64 tb, %2, %9;\n\t"
      "@e_q tcgen05.mma.cta_group::1.kind::f16 [%0], [ra], tb, %3, 1;\n\t"
      "setp.gt.s32 q, %5, 5; and.pred e_q, e, q;\n\t"
      "add.s32 ra, %1, 40; add.s64 tb, %2, %10;\n\t"
      "@e_q tcgen05.mma.cta_group::1.kind::f16 [%0], [ra], tb, %3, 1;\n\t"
      "setp.gt.s32 q, %5, 6; and.pred e_q, e, q;\n\t"
      "add.s32 ra, %1, 48; add.s64 tb, %2, %11;\n\t"
      "@e_q tcgen05.mma.cta_group::1.kind::f16 [%0], [ra], tb, %3, 1;\n\t"
      "setp.gt.s32 q, %5, 7; and.pred e_q, e, q;\n\t"
      "add.s32 ra, %1, 56; add.s64 tb, %2, %12;\n\t"
      "@e_q tcgen05.mma.cta_group::1.kind::f16 [%0], [ra], tb, %3, 1;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(ksteps), "n"(kBStep), "n"(2 * kBStep),
      "n"(3 * kBStep), "n"(4 * kBStep), "n"(5 * kBStep), "n"(6 * kBStep), "n"(7 * kBStep)
      : "memory");
}

__device__ __forceinline__ void mma_commit_elect(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx_elect(uint32_t bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;\n\t}" ::"r"(bar),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d_elect(uint32_t dst, const CUtensorMap* m, uint32_t bar,
                                                  int32_t c0, int32_t c1, int32_t c2) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];\n\t}" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 consecutive 32-bit columns; thread i of the warp gets lane (base lane + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns; thread i of the warp writes lane (base lane + i).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// After tmem_wait_ld: tell the compiler the registers are (re)defined here, so no
// use of them is scheduled above the wait.  Emits no instruction.
template <int N>
__device__ __forceinline__ void reg_fence(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

// ---------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor (tcgen05 "version 1"), 128-byte swizzle.
//   bits  0-13 start address >> 4
//   bits 16-29 leading-dimension byte offset >> 4
//   bits 32-45 stride-dimension byte offset >> 4
//   bits 46-47 version = 1
//   bits 49-51 base offset = 0 (tiles are 1024-byte aligned)
//   bit  52    LBO mode = 0
//   bits 61-63 layout = 2 (SWIZZLE_128B)
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Instruction descriptor for kind::f16 with bf16 A/B and fp32 D.
//   bits 4-5 D format (1 = f32), 7-9 A format (1 = bf16), 10-12 B format (1 = bf16),
//   bit 15 A major (0 = K), bit 16 B major (1 = MN), bits 17-22 N>>3, bits 24-28 M>>4.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn_major ? (1u << 16) : 0u) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// ---------------------------------------------------------------- math
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Three-input maximum (one instruction on sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Packed fp32 pairs (one instruction for two lanes' worth of work): the pair
// lives in one 64-bit register, .x in the low half.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

}  // namespace skptx
