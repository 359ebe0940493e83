// lt_ptx.cuh -- thin inline-PTX wrappers for sm_100a: mbarriers with
// bounded waits, TMA tile loads, tcgen05 (TMEM alloc, MMA, commit, loads)
// and the shared-memory matrix descriptors the tensor cores read.
//
// Everything here is hand-written from the PTX ISA's instruction
// definitions; the descriptor bit positions follow the sm_100 UMMA
// descriptor formats.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <cooperative_groups.h>
#include <cuda_runtime_api.h>  // CUDART_VERSION

// grid_arrive / grid_wait (below) use the barrier word of the cooperative-groups grid
// workspace and its arrive protocol as the CUDA 12.8 / 12.9 headers define
// them; another toolkit may change either, so it must be re-checked there.
static_assert(CUDART_VERSION >= 12080 && CUDART_VERSION < 12100,
              "grid_arrive / grid_wait follow the cooperative-groups grid workspace of CUDA 12.8-12.9");

namespace lt {

// ----------------------------------------------------------------- errors
// Device-side error codes written to the caller-visible error word.
enum : int {
  kDevErrNone = 0,
  kDevErrTimeout = 1,     // a bounded wait gave up (pipeline stalled)
  kDevErrBadSeqlens = 2,  // cu_seqlens not monotone / out of range
};

__device__ __forceinline__ void report_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------- mbarriers
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of the phase of `bar` with the given parity (for a
// thread that polls several barriers).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase of `bar` with the given parity to complete.  The wait
// is bounded: it gives up when *abort becomes non-zero (another role gave
// up) or after `limit_ns` of wall time, in which case it raises *abort,
// records a timeout in the error word and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int* err, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort) return false;
      if (global_timer_ns() - t0 > limit_ns) {
        *abort = 1;
        report_error(err, kDevErrTimeout);
        return false;
      }
    }
  }
}

// ------------------------------------------------------------ named bars
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the
// async proxy (TMA, tensor cores).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------- TMA
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 3-D tiled load into this CTA's shared memory, completing `bytes` on bar.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// 3-D tiled store from this CTA's shared memory (coordinates must not be
// negative; rows past the tensor's extent are not written), tracked in the
// thread's bulk async-group.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0,
                                             int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];"
      ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, const void* src, int c0,
                                             int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];"
      ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2),
      "r"(c3)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// wait until every committed bulk store of this thread has completed
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// wait until every committed bulk store of this thread but the most recent
// one has read its source
__device__ __forceinline__ void bulk_wait_read_but_last() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

// -------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
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

// D[tmem] (+)= A[smem desc] * B[smem desc], kind::f16 (bf16 in, fp32 acc).
__device__ __forceinline__ void umma_f16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16.  A is K-major in TMEM:
// row m in lane m, two consecutive bf16 K elements per 32-bit column (the
// even element in the low half).
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive (once) on bar when every tcgen05.mma issued so far by this thread
// has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 bits, 16 consecutive columns: thread t of the warp receives
// lane (base lane + t), columns [col, col+16).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&r)[16]) {
  uint32_t* u = reinterpret_cast<uint32_t*>(r);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]),
        "=r"(u[7]), "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]),
        "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
      : "r"(taddr));
}

// 32 lanes x 32 bits, 16 consecutive columns, register -> TMEM.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}

// 32 lanes x 32 bits, one column.
__device__ __forceinline__ float tmem_ld1(uint32_t taddr) {
  uint32_t u;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(u) : "r"(taddr));
  return __uint_as_float(u);
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&r)[32]) {
  uint32_t* u = reinterpret_cast<uint32_t*>(r);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]),
        "=r"(u[7]), "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]),
        "=r"(u[13]), "=r"(u[14]), "=r"(u[15]), "=r"(u[16]), "=r"(u[17]), "=r"(u[18]),
        "=r"(u[19]), "=r"(u[20]), "=r"(u[21]), "=r"(u[22]), "=r"(u[23]), "=r"(u[24]),
        "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]), "=r"(u[30]),
        "=r"(u[31])
      : "r"(taddr));
}

// --------------------------------------------- shared-memory descriptors
// Matrix descriptor for a tensor-core operand in shared memory, 128-byte
// swizzle.  Fields: start address >> 4 in bits [0,14), leading byte offset
// >> 4 in [16,30), stride byte offset >> 4 in [32,46), descriptor version 1
// in [46,48), base offset 0, layout type 2 (128-byte swizzle) in [61,64).
//
// K-major operand (rows of the M/N index, K contiguous): rows are 128 B,
// 8-row groups are `sbo` bytes apart; lbo is unused (set to 16 B).
// MN-major operand (rows of the K index, M/N contiguous): each 128-byte row
// holds 64 bf16 of the M/N index; 8-row K groups are `sbo` bytes apart and
// successive 64-element M/N groups are `lbo` bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// The same descriptor with its start address advanced by `bytes` (the
// start-address field holds addr >> 4 in 14 bits; shared addresses stay
// below 256 KB, so the add never carries out of the field).
__device__ __forceinline__ uint64_t desc_advance(uint64_t desc, uint32_t bytes) {
  return desc + (uint64_t)(bytes >> 4);
}

// Instruction descriptor for kind::f16 with bf16 A/B and fp32 accumulator.
// a_mn / b_mn: 1 when the operand is MN-major, 0 when K-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                            // D format: f32
         | (1u << 7)                          // A format: bf16
         | (1u << 10)                         // B format: bf16
         | ((uint32_t)a_mn << 15)             // A major
         | ((uint32_t)b_mn << 16)             // B major
         | ((uint32_t)(N >> 3) << 17)         // N / 8
         | ((uint32_t)(M >> 4) << 24);        // M / 16
}

// ------------------------------------------------------------ conversions
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Hardware base-2 exponential (MUFU), fp32 in and out.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Feature map on a pair of packed bf16 values, phi(x) = ELU(x) + 1:
// x + 1 for x > 0, e^x = 2^(x log2 e) otherwise, each evaluated in fp32 and
// rounded once to bf16 (the precision of the tensor-core operand).  The
// exponential is taken for every x and discarded for x > 0 (where it may
// overflow to +inf); NaN propagates through the exponential.
__device__ __forceinline__ uint32_t phi_bf16x2(uint32_t x) {
  const float lo = __uint_as_float(x << 16), hi = __uint_as_float(x & 0xFFFF0000u);
  const float elo = ex2_approx(lo * 1.4426950408889634f);
  const float ehi = ex2_approx(hi * 1.4426950408889634f);
  return pack_bf16x2(lo > 0.0f ? lo + 1.0f : elo, hi > 0.0f ? hi + 1.0f : ehi);
}

// ------------------------------------------------ kernel variants
// Input element type and feature map of a forward kernel, as compile-time
// parameters.  Var<kInBf16, kPhiElu1> is the method's default (bf16 I/O,
// phi = ELU + 1) and compiles to the code above.  The tensor-core operands
// are bf16 for every variant: fp16 inputs are widened exactly to fp32,
// transformed, and rounded once to bf16 (V included); outputs take the
// input's type.
enum : int { kInBf16 = 0, kInF16 = 1 };
enum : int { kPhiElu1 = 0, kPhiRelu = 1, kPhiExp = 2 };

template <int IN, int PHI>
struct Var {
  static constexpr int kIn = IN;
  static constexpr int kPhi = PHI;
  static constexpr bool kDefault = IN == kInBf16 && PHI == kPhiElu1;
};
using VarDefault = Var<kInBf16, kPhiElu1>;

// two packed 16-bit input elements -> fp32 (the even element in the low half)
template <int IN>
__device__ __forceinline__ float2 unpack_in(uint32_t u) {
  if constexpr (IN == kInBf16) {
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
  } else {
    __half2 h = *reinterpret_cast<__half2*>(&u);
    return __half22float2(h);
  }
}

// the feature maps, fp32 in and out: ELU + 1 (x + 1 for x > 0, e^x else),
// ReLU (max(x, 0)), exp (e^x); e^x as 2^(x log2 e) on the MUFU
template <int PHI>
__device__ __forceinline__ float feat(float x) {
  if constexpr (PHI == kPhiElu1) {
    const float e = ex2_approx(x * 1.4426950408889634f);
    return x > 0.0f ? x + 1.0f : e;
  } else if constexpr (PHI == kPhiRelu) {
    return fmaxf(x, 0.0f);
  } else {
    return ex2_approx(x * 1.4426950408889634f);
  }
}

// phi on two packed inputs -> two packed bf16 operands
template <class V>
__device__ __forceinline__ uint32_t phi2(uint32_t x) {
  if constexpr (V::kDefault) {
    return phi_bf16x2(x);
  } else {
    const float2 f = unpack_in<V::kIn>(x);
    return pack_bf16x2(feat<V::kPhi>(f.x), feat<V::kPhi>(f.y));
  }
}

// two packed inputs (V tiles) -> two packed bf16 operands
template <class V>
__device__ __forceinline__ uint32_t conv2(uint32_t x) {
  if constexpr (V::kIn == kInBf16) {
    return x;
  } else {
    const float2 f = unpack_in<V::kIn>(x);
    return pack_bf16x2(f.x, f.y);
  }
}

// two fp32 results -> two packed outputs of the input's type
template <class V>
__device__ __forceinline__ uint32_t pack_out(float lo, float hi) {
  if constexpr (V::kIn == kInBf16) {
    return pack_bf16x2(lo, hi);
  } else {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
}

// ------------------------------------------------------------ grid barrier
// Grid-wide barrier of a cooperative launch, on the barrier word the driver
// provides to such a launch (the word and the flip-bit protocol of the
// cooperative-groups grid synchronisation: every CTA adds 1 and block
// (0,0,0) adds 2^31 - (ctas - 1), so the top bit flips once every CTA has
// arrived and the low bits return to their former value), in two parts for a
// CTA that arrives early and waits later.  grid_arrive: one thread per CTA,
// exactly once per CTA and launch, on every path; it stores the barrier
// word's value before the arrival in *old and returns false (after recording
// an error) when the launch is not cooperative.  grid_wait(old): wait,
// bounded like mbar_wait, until every CTA has arrived.
__device__ __forceinline__ bool grid_arrive(unsigned int* old, volatile int* abort, int* err) {
  cooperative_groups::details::grid_workspace* gw =
      cooperative_groups::details::get_grid_workspace();
  if (gw == nullptr) {
    *abort = 1;
    report_error(err, kDevErrTimeout);
    return false;
  }
  const unsigned int ctas = gridDim.x * gridDim.y * gridDim.z;
  const bool master = (blockIdx.x | blockIdx.y | blockIdx.z) == 0;
  const unsigned int inc = master ? 0x80000000u - (ctas - 1u) : 1u;
  unsigned int o;
  asm volatile("atom.add.release.gpu.u32 %0, [%1], %2;" : "=r"(o) : "l"(&gw->barrier), "r"(inc)
               : "memory");
  *old = o;
  return true;
}

__device__ __forceinline__ bool grid_wait(unsigned int old, volatile int* abort, int* err,
                                          uint64_t limit_ns) {
  cooperative_groups::details::grid_workspace* gw =
      cooperative_groups::details::get_grid_workspace();
  unsigned int* bar = &gw->barrier;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    unsigned int cur;
    asm volatile("ld.acquire.gpu.u32 %0, [%1];" : "=r"(cur) : "l"(bar) : "memory");
    if ((cur ^ old) & 0x80000000u) return true;
    if (*abort) return false;
    if (global_timer_ns() - t0 > limit_ns) {
      *abort = 1;
      report_error(err, kDevErrTimeout);
      return false;
    }
    __nanosleep(128);  // one poller per CTA on one word: keep its line cool
  }
}

}  // namespace lt
