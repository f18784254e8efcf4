// Hand-written inline-PTX wrappers for sm_100a: mbarriers with bounded waits,
// TMA tile loads (no multicast), tcgen05 tensor-memory allocation, MMA, commit,
// loads and stores.  Only what the h3attn kernels use.
#pragma once
#include <cstdint>

namespace h3 {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint64_t clock_now() {
  uint64_t c;
  asm volatile("mov.u64 %0, %clock64;" : "=l"(c));
  return c;
}

// ------------------------------------------------------------- mbarrier ----
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of the phase with the given parity (acquire at CTA scope on
// success): its latency overlaps whatever the thread issues before it uses the result.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait that lets the hardware suspend the thread for up to hint_ns while
// the phase is incomplete (it resumes when the phase completes), so waiting
// warps do not spin on the issue slots the working warps need.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity.  Returns false if the wait
// gave up: after `limit_ns` of global time, or soon after *abort (a CTA-wide
// flag in shared memory; may be null) becomes non-zero.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const volatile int* abort,
                                          uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, 100000u)) return true;  // up to 0.1 ms per try
    if (abort != nullptr && *abort) return false;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (tensor-core operand reads) ordered after a later barrier arrive.
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ------------------------------------------------------------------ TMA ----
// 2D tiled bulk tensor load global -> shared, completion on an mbarrier (tx bytes).
// No cluster multicast.  x is the innermost coordinate (bytes for 8-bit data).
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          smem_u32(dst)),
      "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// -------------------------------------------------------------- tcgen05 ----
// Tensor memory address: bits 31..16 lane, bits 15..0 column.
__device__ __forceinline__ void tmem_alloc(uint32_t* holder_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(holder_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] x B[smem desc]^T, E4M3 operands, F32 accumulate.
__device__ __forceinline__ void mma_f8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[smem desc] x B[smem desc]^T, BF16 operands, F32 accumulate.
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 bits, 32 consecutive columns: thread i gets lane (base + i).
// The load and its wait are one asm statement, so no use of r[] can be
// scheduled before the data has arrived.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// 32 lanes x 32 bits, 64 consecutive columns into r[OFF, OFF + 64), load and wait
// in one statement.
template <int OFF>
__device__ __forceinline__ void tmem_ld64_wait_at(uint32_t taddr, uint32_t (&r)[128]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[OFF + 0]), "=r"(r[OFF + 1]), "=r"(r[OFF + 2]), "=r"(r[OFF + 3]), "=r"(r[OFF + 4]), "=r"(r[OFF + 5]), "=r"(r[OFF + 6]), "=r"(r[OFF + 7]), "=r"(r[OFF + 8]), "=r"(r[OFF + 9]), "=r"(r[OFF + 10]), "=r"(r[OFF + 11]), "=r"(r[OFF + 12]), "=r"(r[OFF + 13]), "=r"(r[OFF + 14]), "=r"(r[OFF + 15]), "=r"(r[OFF + 16]), "=r"(r[OFF + 17]), "=r"(r[OFF + 18]), "=r"(r[OFF + 19]), "=r"(r[OFF + 20]), "=r"(r[OFF + 21]), "=r"(r[OFF + 22]), "=r"(r[OFF + 23]), "=r"(r[OFF + 24]), "=r"(r[OFF + 25]), "=r"(r[OFF + 26]), "=r"(r[OFF + 27]), "=r"(r[OFF + 28]), "=r"(r[OFF + 29]), "=r"(r[OFF + 30]), "=r"(r[OFF + 31]), "=r"(r[OFF + 32]), "=r"(r[OFF + 33]), "=r"(r[OFF + 34]), "=r"(r[OFF + 35]), "=r"(r[OFF + 36]), "=r"(r[OFF + 37]), "=r"(r[OFF + 38]), "=r"(r[OFF + 39]), "=r"(r[OFF + 40]), "=r"(r[OFF + 41]), "=r"(r[OFF + 42]), "=r"(r[OFF + 43]), "=r"(r[OFF + 44]), "=r"(r[OFF + 45]), "=r"(r[OFF + 46]), "=r"(r[OFF + 47]), "=r"(r[OFF + 48]), "=r"(r[OFF + 49]), "=r"(r[OFF + 50]), "=r"(r[OFF + 51]), "=r"(r[OFF + 52]), "=r"(r[OFF + 53]), "=r"(r[OFF + 54]), "=r"(r[OFF + 55]), "=r"(r[OFF + 56]), "=r"(r[OFF + 57]), "=r"(r[OFF + 58]), "=r"(r[OFF + 59]), "=r"(r[OFF + 60]), "=r"(r[OFF + 61]), "=r"(r[OFF + 62]), "=r"(r[OFF + 63])
      : "r"(taddr)
      : "memory");
}

// The same load without the wait: r[OFF, OFF + 64) is not valid until
// tmem_wait_ld_at<OFF> on the same array, which every use must follow.
template <int OFF>
__device__ __forceinline__ void tmem_ld64_async_at(uint32_t taddr, uint32_t (&r)[128]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
      : "=r"(r[OFF + 0]), "=r"(r[OFF + 1]), "=r"(r[OFF + 2]), "=r"(r[OFF + 3]), "=r"(r[OFF + 4]), "=r"(r[OFF + 5]), "=r"(r[OFF + 6]), "=r"(r[OFF + 7]), "=r"(r[OFF + 8]), "=r"(r[OFF + 9]), "=r"(r[OFF + 10]), "=r"(r[OFF + 11]), "=r"(r[OFF + 12]), "=r"(r[OFF + 13]), "=r"(r[OFF + 14]), "=r"(r[OFF + 15]), "=r"(r[OFF + 16]), "=r"(r[OFF + 17]), "=r"(r[OFF + 18]), "=r"(r[OFF + 19]), "=r"(r[OFF + 20]), "=r"(r[OFF + 21]), "=r"(r[OFF + 22]), "=r"(r[OFF + 23]), "=r"(r[OFF + 24]), "=r"(r[OFF + 25]), "=r"(r[OFF + 26]), "=r"(r[OFF + 27]), "=r"(r[OFF + 28]), "=r"(r[OFF + 29]), "=r"(r[OFF + 30]), "=r"(r[OFF + 31]), "=r"(r[OFF + 32]), "=r"(r[OFF + 33]), "=r"(r[OFF + 34]), "=r"(r[OFF + 35]), "=r"(r[OFF + 36]), "=r"(r[OFF + 37]), "=r"(r[OFF + 38]), "=r"(r[OFF + 39]), "=r"(r[OFF + 40]), "=r"(r[OFF + 41]), "=r"(r[OFF + 42]), "=r"(r[OFF + 43]), "=r"(r[OFF + 44]), "=r"(r[OFF + 45]), "=r"(r[OFF + 46]), "=r"(r[OFF + 47]), "=r"(r[OFF + 48]), "=r"(r[OFF + 49]), "=r"(r[OFF + 50]), "=r"(r[OFF + 51]), "=r"(r[OFF + 52]), "=r"(r[OFF + 53]), "=r"(r[OFF + 54]), "=r"(r[OFF + 55]), "=r"(r[OFF + 56]), "=r"(r[OFF + 57]), "=r"(r[OFF + 58]), "=r"(r[OFF + 59]), "=r"(r[OFF + 60]), "=r"(r[OFF + 61]), "=r"(r[OFF + 62]), "=r"(r[OFF + 63])
      : "r"(taddr)
      : "memory");
}

// Wait for this thread's tensor-memory loads; r[OFF, OFF + 64) (the destination of
// an earlier tmem_ld64_async_at) is an in/out operand, so no use of it can be
// scheduled before the wait.
template <int OFF>
__device__ __forceinline__ void tmem_wait_ld_at(uint32_t (&r)[128]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[OFF + 0]), "+r"(r[OFF + 1]), "+r"(r[OFF + 2]), "+r"(r[OFF + 3]), "+r"(r[OFF + 4]), "+r"(r[OFF + 5]), "+r"(r[OFF + 6]), "+r"(r[OFF + 7]), "+r"(r[OFF + 8]), "+r"(r[OFF + 9]), "+r"(r[OFF + 10]), "+r"(r[OFF + 11]), "+r"(r[OFF + 12]), "+r"(r[OFF + 13]), "+r"(r[OFF + 14]), "+r"(r[OFF + 15]), "+r"(r[OFF + 16]), "+r"(r[OFF + 17]), "+r"(r[OFF + 18]), "+r"(r[OFF + 19]), "+r"(r[OFF + 20]), "+r"(r[OFF + 21]), "+r"(r[OFF + 22]), "+r"(r[OFF + 23]), "+r"(r[OFF + 24]), "+r"(r[OFF + 25]), "+r"(r[OFF + 26]), "+r"(r[OFF + 27]), "+r"(r[OFF + 28]), "+r"(r[OFF + 29]), "+r"(r[OFF + 30]), "+r"(r[OFF + 31]), "+r"(r[OFF + 32]), "+r"(r[OFF + 33]), "+r"(r[OFF + 34]), "+r"(r[OFF + 35]), "+r"(r[OFF + 36]), "+r"(r[OFF + 37]), "+r"(r[OFF + 38]), "+r"(r[OFF + 39]), "+r"(r[OFF + 40]), "+r"(r[OFF + 41]), "+r"(r[OFF + 42]), "+r"(r[OFF + 43]), "+r"(r[OFF + 44]), "+r"(r[OFF + 45]), "+r"(r[OFF + 46]), "+r"(r[OFF + 47]), "+r"(r[OFF + 48]), "+r"(r[OFF + 49]), "+r"(r[OFF + 50]), "+r"(r[OFF + 51]), "+r"(r[OFF + 52]), "+r"(r[OFF + 53]), "+r"(r[OFF + 54]), "+r"(r[OFF + 55]), "+r"(r[OFF + 56]), "+r"(r[OFF + 57]), "+r"(r[OFF + 58]), "+r"(r[OFF + 59]), "+r"(r[OFF + 60]), "+r"(r[OFF + 61]), "+r"(r[OFF + 62]), "+r"(r[OFF + 63])
               :
               : "memory");
}

// A read-only FP32 global load issued where it stands in the program (a volatile asm
// statement): the compiler may not sink it to its first use, so a load issued one loop
// iteration ahead of that use keeps its latency off the iteration's critical path.
__device__ __forceinline__ float ldg_f32_issued_here(const float* ptr) {
  float v;
  asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(ptr) : "memory");
  return v;
}

// ------------------------------------------------------ packed FP32 pairs ----
// sm_100 f32x2 instructions: two IEEE FP32 operations (round to nearest even,
// subnormals kept) per instruction on a 64-bit register pair.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
// Maximum of three FP32 values.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// Warpgroup register reallocation (all four warps of a warpgroup execute it).
template <uint32_t kRegs>
__device__ __forceinline__ void regs_dealloc() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegs));
}
template <uint32_t kRegs>
__device__ __forceinline__ void regs_alloc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegs));
}

// --------------------------------------------------- UMMA descriptors ----
// Shared-memory matrix descriptor for a K-major operand tile stored with the
// 128-byte swizzle: rows of 128 bytes, 8-row atoms of 1024 bytes (stride byte
// offset), tile base aligned to 1024 bytes.  Fields: start address >> 4 in
// bits 0-13, leading byte offset >> 4 in 16-29 (unused for this layout, 1),
// stride byte offset >> 4 in 32-45, descriptor version 1 in 46-47, swizzle
// mode in 61-63 (2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t sdesc_k_sw128(uint32_t smem_addr) {
  return (uint64_t)((smem_addr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor: D format in bits 4-5 (1 = F32), A format in 7-9, B format in
// 10-12 (FP8: 0 = E4M3; 16-bit: 1 = BF16), both operands K-major (bits 15, 16 = 0),
// N >> 3 in 17-22, M >> 4 in 24-28.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ------------------------------------------------------------ numerics ----
// Two FP32 -> packed E4M3x2 (round to nearest even, saturate to +-448);
// `lo` lands in the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return (uint32_t)r;
}

// Four FP32 -> four E4M3 in one instruction, a in the low byte: the 4-wide conversion
// with its rounding bits fixed at one half step for every element (0x8001 in each
// 16-bit half: bit 15 is the top rounding bit of the first element of the half, bit 0
// that of the second, whose bits run in the opposite order), i.e. round to nearest
// with ties away from zero, saturating to +-448.  It differs from
// cvt_e4m3x2 (ties to even) only at exact ties and for values within 2^-16 of a
// step below a midpoint.
__device__ __forceinline__ uint32_t cvt_e4m3x4_half_up(float a, float b, float c, float d) {
  uint32_t r;
  asm("cvt.rs.satfinite.e4m3x4.f32 %0, {%1, %2, %3, %4}, %5;" : "=r"(r) : "f"(d), "f"(c), "f"(b), "f"(a),
      "r"(0x80018001u));
  return r;
}

}  // namespace h3
