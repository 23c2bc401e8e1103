// Device primitives for sm_100a: mbarriers, TMA tile loads, tcgen05 (UMMA)
// issue / commit, tensor-memory allocation and loads/stores, and the shared
// memory and instruction descriptors the tensor cores read.
//
// Everything here is a thin inline-PTX wrapper written from the PTX ISA
// descriptions of these instructions. No cluster multicast is used anywhere:
// every CTA fetches its own tiles.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace fa {

// ---------------------------------------------------------------------------
// error word shared by all kernels of the library (bounded waits write here)
// ---------------------------------------------------------------------------
enum : int {
  kDevOk = 0,
  kDevTimeout = 1,
};
// The library is built as one translation unit, so a file-scope variable is
// shared by every kernel and by the host code that reads it back.
static __device__ int g_device_status = 0;
// which bounded wait gave up first (0 = none): 100 * kernel + wait, for the
// error message of fa_get_device_status
static __device__ int g_wait_site = 0;

__device__ __forceinline__ void record_timeout(int site) {
  atomicExch(&g_device_status, 1 /* kDevTimeout */);
  if (site != 0) atomicCAS(&g_wait_site, 0, site);
}

// Bounded waits give up after this many nanoseconds of %globaltimer.
constexpr uint64_t kWaitTimeoutNs = 4000000000ull;  // 4 s

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t lane_id() { return threadIdx.x & 31u; }

__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
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

// Wait for the phase with the given parity to complete. Returns false (and
// records kDevTimeout in the library's device status word) if it has not
// completed within kWaitTimeoutNs; the caller then unwinds instead of hanging.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          uint64_t limit_ns = kWaitTimeoutNs, int site = 0) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0u && globaltimer_ns() - t0 > limit_ns) {
      record_timeout(site);
      return false;
    }
  }
}

// ---------------------------------------------------------------------------
// fences
// ---------------------------------------------------------------------------
// make generic-proxy shared-memory writes visible to the async proxy
// (tcgen05.mma operand reads, TMA stores)
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Per-warpgroup register reallocation. All four warps of a warpgroup execute
// it. The block's pool is fixed at launch (threads x registers at launch), so
// the sum of the warpgroups' new limits must stay within it, or inc waits.
template <uint32_t kRegs>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegs));
}
template <uint32_t kRegs>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegs));
}

// named barrier over a subset of warps (id 1..15; 0 is __syncthreads)
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------
// TMA (no multicast)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(const CUtensorMap* map, uint64_t* bar, void* dst,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(const CUtensorMap* map, uint64_t* bar, void* dst,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Untiled bulk copy of `bytes` from global to this CTA's shared memory,
// completing on `bar` (no multicast). Both addresses 16-byte aligned, bytes
// a multiple of 16.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory
// ---------------------------------------------------------------------------
// Whole warp. Writes the allocated TMEM base address to *dst (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst)),
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

// TMEM address: lane in bits [31:16], column in [15:0]
__device__ __forceinline__ uint32_t tmem_addr(uint32_t base, uint32_t lane, uint32_t col) {
  return base + (lane << 16) + col;
}

#define FA_R8(i) "=r"(r[i + 0]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), \
                 "=r"(r[i + 4]), "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
#define FA_W8(i) "r"(r[i + 0]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), \
                 "r"(r[i + 4]), "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])

// 32 lanes x 32 bit, 16 consecutive columns per thread (thread t <-> lane base+t)
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : FA_R8(0), FA_R8(8)
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : FA_R8(0), FA_R8(8), FA_R8(16), FA_R8(24)
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      FA_W8(0), FA_W8(8)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      FA_W8(0), FA_W8(8), FA_W8(16), FA_W8(24)
      : "memory");
}
#undef FA_R8
#undef FA_W8

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: MMA (issued by one thread)
// ---------------------------------------------------------------------------
// D[tmem] (+)= A[smem desc] * B[smem desc]
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// kind::f8f6f4 forms of the two above (both operands 8-bit, here E4M3; the
// instruction descriptor names the formats)
__device__ __forceinline__ void umma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

template <bool kF8>
__device__ __forceinline__ void umma_ss_k(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
  if constexpr (kF8) umma_ss_f8(d, a, b, id, acc); else umma_ss(d, a, b, id, acc);
}
template <bool kF8>
__device__ __forceinline__ void umma_ts_k(uint32_t d, uint32_t a, uint64_t b, uint32_t id, uint32_t acc) {
  if constexpr (kF8) umma_ts_f8(d, a, b, id, acc); else umma_ts(d, a, b, id, acc);
}

// Arrive once on *bar when every tcgen05 async op issued so far by this
// thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------------------
// descriptors
// ---------------------------------------------------------------------------
// Shared-memory matrix descriptor, 128-byte swizzle (the layout TMA writes
// with CU_TENSOR_MAP_SWIZZLE_128B). Byte offsets are encoded >> 4.
//   K-major operand:  rows of 128 B (64 16-bit elements of K), 8-row swizzle
//                     atoms `sbo` bytes apart; `lbo` unused.
//   MN-major operand: rows of 128 B (64 16-bit elements of M or N) indexed by
//                     K; 8-K-row atoms `sbo` apart, 64-wide M/N chunks `lbo` apart.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;  // descriptor version for sm_100
  d |= static_cast<uint64_t>(2) << 61;  // 128-byte swizzle
  return d;
}

// Instruction descriptor for kind::f8f6f4 with E4M3 A and B (format code 0
// in both fields) and fp32 accumulation; the other fields as idesc_f16.
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Instruction descriptor for kind::f16 with fp32 accumulation.
__host__ __device__ constexpr uint32_t idesc_f16(bool bf16, int M, int N, bool a_mn_major,
                                                 bool b_mn_major) {
  return (1u << 4)                                  // D format: f32
         | ((bf16 ? 1u : 0u) << 7)                  // A format: f16 / bf16
         | ((bf16 ? 1u : 0u) << 10)                 // B format
         | ((a_mn_major ? 1u : 0u) << 15)           // A major
         | ((b_mn_major ? 1u : 0u) << 16)           // B major
         | (static_cast<uint32_t>(N >> 3) << 17)    // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);   // M / 16
}

// ---------------------------------------------------------------------------
// small numeric helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x for a pair of values on the FMA and integer pipes instead of the
// special-function unit. x = n + f with n = round(x) (adding 1.5 * 2^23
// rounds to an integer held in the low mantissa bits) and f in [-1/2, 1/2];
// 2^f is a cubic fitted for minimal relative error by the Remez exchange
// algorithm (fit_polynomials.py next to this file; float32 relative error
// 7.5e-5), and n is added into the exponent field: the low 9 bits of the
// rounded value's bit pattern, shifted by 23, are n << 23 modulo 2^32.
// x is clamped at -125 so that the result's exponent field stays >= 1 (at
// n = -126 a cubic below 1 would land on the subnormal encoding, which the
// bit addition does not produce correctly): smaller inputs (masked logits,
// -inf) give a value near 2^-125 rather than 0.
__device__ __forceinline__ float2 ex2_poly2(float2 x) {
  x.x = fmaxf(x.x, -125.f);
  x.y = fmaxf(x.y, -125.f);
  const float2 j = __fadd2_rn(x, make_float2(12582912.f, 12582912.f));
  const float2 n = __fadd2_rn(j, make_float2(-12582912.f, -12582912.f));
  const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);
  float2 q = __ffma2_rn(f, make_float2(5.517166906e-02f, 5.517166906e-02f),
                        make_float2(2.426111222e-01f, 2.426111222e-01f));
  q = __ffma2_rn(q, f, make_float2(6.932609855e-01f, 6.932609855e-01f));
  q = __ffma2_rn(q, f, make_float2(9.999280735e-01f, 9.999280735e-01f));
  return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(j.x) << 23)),
                     __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(j.y) << 23)));
}

// tanh from the identity tanh(y) = sign(y) (1 - e) / (1 + e), e = exp(-2|y|),
// with e taken as 2^(-2 |y| log2(e)). Absolute error ~2e-7 (the subtraction
// 1 - e near y = 0 and the exp2/rcp approximations); with softcap c the
// logit error is ~c * 2e-7.
__device__ __forceinline__ float tanh_fast(float y) {
  const float e = ex2_approx(fabsf(y) * -2.8853900817779268f);
  return copysignf(__fdividef(1.f - e, 1.f + e), y);
}

// tanh(y) = y * Q(y^2) for |y| <= kTanhPolyMax, Q of degree 4 fitted by the
// Remez exchange algorithm for minimal relative error (fit_polynomials.py next
// to this file derives the coefficients; float64 relative error 1.3e-8,
// float32 evaluation within 4e-8 absolute). Two values per call, on the FMA
// pipe, instead of the two special-function operations of tanh_fast.
constexpr float kTanhPolyMax = 0.5f;
__device__ __forceinline__ float2 tanh_poly2(float2 y) {
  const float2 t = __fmul2_rn(y, y);
  float2 q = __ffma2_rn(make_float2(1.713500663e-02f, 1.713500663e-02f), t,
                        make_float2(-5.298607529e-02f, -5.298607529e-02f));
  q = __ffma2_rn(q, t, make_float2(1.332477932e-01f, 1.332477932e-01f));
  q = __ffma2_rn(q, t, make_float2(-3.333306939e-01f, -3.333306939e-01f));
  q = __ffma2_rn(q, t, make_float2(9.999999869e-01f, 9.999999869e-01f));
  return __fmul2_rn(y, q);
}

// c * tanh(a * x) for a pair of values, as x * P(x^2) with the fitted
// coefficients q_k of tanh(y) = y Q(y^2) folded into P_k = c a^(2k+1) q_k
// (fold_tanh), so that the scale, the softcap division and multiplication
// and the tanh together cost one multiply and kN FMAs per pair.
// kTanhLo: degree 2 for |a x| <= kTanhPolyMaxLo (Remez, fit_polynomials.py;
// float64 relative error 4.0e-7, float32 evaluation within 1.1e-7 absolute).
// kTanhHi: the degree-4 coefficients of tanh_poly2, |a x| <= kTanhPolyMax.
// kTanhCubic: degree 1 (tanh as an odd cubic) for |a x| <= kTanhCubicMax
// (Remez, fit_polynomials.py; float64 relative error 4.0e-6, float32
// evaluation within 5.1e-7 absolute).
constexpr float kTanhPolyMaxLo = 0.25f;
constexpr float kTanhCubicMax = 0.125f;
__device__ constexpr float kTanhCubic[2] = {9.999959588e-01f, -3.312617543e-01f};
__device__ constexpr float kTanhLo[3] = {9.999996043e-01f, -3.332190823e-01f, 1.284161343e-01f};
__device__ constexpr float kTanhHi[5] = {9.999999869e-01f, -3.333306939e-01f, 1.332477932e-01f,
                                         -5.298607529e-02f, 1.713500663e-02f};

template <int kN>
__device__ __forceinline__ void fold_tanh(const float (&q)[kN], float a, float c, float (&pk)[kN]) {
  float f = c * a;
  const float a2 = a * a;
#pragma unroll
  for (int k = 0; k < kN; ++k) {
    pk[k] = f * q[k];
    f *= a2;
  }
}

template <int kN>
__device__ __forceinline__ float2 tanh_fold2(float2 x, const float (&pk)[kN]) {
  const float2 u = __fmul2_rn(x, x);
  float2 r = make_float2(pk[kN - 1], pk[kN - 1]);
#pragma unroll
  for (int k = kN - 2; k >= 0; --k) r = __ffma2_rn(r, u, make_float2(pk[k], pk[k]));
  return __fmul2_rn(x, r);
}

template <bool kBF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (kBF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
}

// Two finite floats -> packed 16-bit pair like pack2, but for bf16 on the
// integer pipe: add half a bf16 ulp (0x8000) to each bit pattern and keep the
// high halves (one prmt). That rounds half away from zero instead of to even:
// the same half-ulp error bound, different only on exact ties. The
// conversion instruction shares its unit with ex2, which the softmax keeps
// busy; fp16 keeps the conversion.
template <bool kBF16>
__device__ __forceinline__ uint32_t pack2_alu(float lo, float hi) {
  if constexpr (kBF16) {
    const uint32_t a = __float_as_uint(lo) + 0x8000u;
    const uint32_t b = __float_as_uint(hi) + 0x8000u;
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(r) : "r"(a), "r"(b));
    return r;
  } else {
    return pack2<false>(lo, hi);
  }
}

// Four non-negative floats -> four FP8 E4M3 bytes, x0 in the lowest byte
// (round to nearest even, saturating at 448). The conversion instruction
// takes two floats and writes its first source into the upper byte.
__device__ __forceinline__ uint32_t pack4_e4m3(float x0, float x1, float x2, float x3) {
  uint32_t lo, hi;
  asm("{\n\t.reg .b16 t;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\t"
      "cvt.u32.u16 %0, t;\n\t}" : "=r"(lo) : "f"(x1), "f"(x0));
  asm("{\n\t.reg .b16 t;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\t"
      "cvt.u32.u16 %0, t;\n\t}" : "=r"(hi) : "f"(x3), "f"(x2));
  return lo | (hi << 16);
}

template <bool kBF16>
__device__ __forceinline__ float2 unpack2(uint32_t u) {
  if constexpr (kBF16) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
    return __bfloat1622float2(v);
  } else {
    __half2 v = *reinterpret_cast<__half2*>(&u);
    return __half22float2(v);
  }
}

}  // namespace fa
