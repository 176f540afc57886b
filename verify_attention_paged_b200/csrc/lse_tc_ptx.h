// Inline-PTX helpers shared by the tensor-core (tcgen05) kernels of
// liblse_attn.so: mbarrier waits with a time limit, TMA and bulk copies,
// UMMA shared-memory and instruction descriptors, tcgen05 MMA issue and
// commit, TMEM loads and stores, fast exp2/log2/reciprocal, and the
// conversions of FP32 values into the 16-bit and 8-bit operand terms the
// products take.  Not part of the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "lse_attn.h"

namespace lse_ptx {

// Every bounded wait gives up after this many SM clock cycles (~2 s at
// 2 GHz) and reports LSE_DEVERR_TIMEOUT.
constexpr long long kWaitCycles = 4000000000ll;

__device__ __forceinline__ uint32_t smem_u32(const void *ptr) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(ptr));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
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

// As mbar_try_wait, but a thread whose phase is not complete is suspended
// (until the phase completes, or for at most about a microsecond) instead of
// returning at once, so waiting warps leave their issue slots to the warps
// doing work.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "n"(1000)
      : "memory");
  return ok != 0;
}

// Slow path of mbar_wait (out of line: it runs only when the phase is not
// complete at the first test).
static __device__ __noinline__ bool mbar_wait_spin(uint32_t bar, uint32_t parity,
                                            volatile int *abort_flag, unsigned int *err) {
  const long long t0 = clock64();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait_sleep(bar, parity)) return true;
    if ((i & 3u) == 0) {
      if (*abort_flag) return false;
      if (clock64() - t0 > kWaitCycles) {
        *abort_flag = 1;
        atomicOr(err, LSE_DEVERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Wait for the phase of `bar` with the given parity; false when the wait ran
// out (then the CTA-wide abort flag is set) or another role aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                          unsigned int *err) {
  return mbar_try_wait(bar, parity) || mbar_wait_spin(bar, parity, abort_flag, err);
}

// Time-bounded wait that ignores the abort flag: used to drain copies and
// MMAs already in flight before the CTA releases TMEM and exits.
static __device__ __noinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait_sleep(bar, parity))
    if (clock64() - t0 > kWaitCycles) return;
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ bool named_or(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred a, b;\n\t"
      "setp.ne.u32 a, %1, 0;\n\t"
      "bar.red.or.pred b, %2, %3, a;\n\t"
      "selp.u32 %0, 1, 0, b;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Plain bulk copy global -> shared (no tensor map, no multicast), counted
// on an mbarrier's transaction bytes.  Both addresses 16-byte aligned, bytes
// a multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// UMMA shared-memory matrix descriptor.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
}
constexpr uint32_t kLayoutNone = 0;
constexpr uint32_t kLayoutSw128 = 2;

// Instruction descriptor, FP32 accumulation.  Formats: kind::f16 takes
// 0 = F16, 1 = BF16 (A and B alike); kind::f8f6f4 takes 0 = E4M3, 1 = E5M2
// for A and B independently.  a_mn / b_mn: 1 = MN-major operand.
__host__ __device__ constexpr uint32_t instr_desc(uint32_t a_fmt, uint32_t b_fmt, uint32_t a_mn,
                                                  uint32_t b_mn, uint32_t M, uint32_t N) {
  return (1u << 4) | (a_fmt << 7) | (b_fmt << 10) | (a_mn << 15) | (b_mn << 16) |
         ((N >> 3) << 17) | ((M >> 4) << 24);
}

// One lane of the warp (elect.sync): 1 in that lane, 0 in the others.
__device__ __forceinline__ uint32_t elect_one() {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred e;\n\t.reg .b32 x;\n\t"
      "elect.sync x|e, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, e;\n\t}\n"
      : "=r"(r));
  return r;
}

// The MMA issue helpers run in all lanes of a converged warp with the same
// operands; only the lane with `leader` set issues.
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                        uint32_t accumulate, uint32_t leader) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.ne.b32 e, %5, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(leader)
      : "memory");
}
// 8-bit operands, K = 32 per instruction.
__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t accumulate, uint32_t leader) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.ne.b32 e, %5, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(leader)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar, uint32_t leader) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "setp.ne.b32 e, %1, 0;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}\n" ::"r"(bar),
      "r"(leader)
      : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float *v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(
          taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two FP32 values -> packed hi (nearest 16-bit) and lo (its rounding error).
template <int DT>
__device__ __forceinline__ void split2(float x0, float x1, uint32_t &hi, uint32_t &lo);
template <>
__device__ __forceinline__ void split2<LSE_KV_BF16>(float x0, float x1, uint32_t &hi,
                                                    uint32_t &lo) {
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(hi) : "f"(x1), "f"(x0));
  const float h0 = __uint_as_float(hi << 16), h1 = __uint_as_float(hi & 0xffff0000u);
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(lo) : "f"(x1 - h1), "f"(x0 - h0));
}
template <>
__device__ __forceinline__ void split2<LSE_KV_F16>(float x0, float x1, uint32_t &hi,
                                                   uint32_t &lo) {
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(hi) : "f"(x1), "f"(x0));
  const float2 h = __half22float2(*reinterpret_cast<const __half2 *>(&hi));
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(lo) : "f"(x1 - h.y), "f"(x0 - h.x));
}

// Two FP32 values -> the nearest 8-bit pair (x1 in the high byte, saturating
// at the format's largest finite value), and the values that pair decodes
// to (exactly, through F16, which holds every E4M3 and E5M2 value).
template <bool kE5>
__device__ __forceinline__ uint32_t f8x2(float x0, float x1, float &d0, float &d1) {
  uint16_t r;
  uint32_t h;
  if (kE5) {
    asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(x1), "f"(x0));
    asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(h) : "h"(r));
  } else {
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(x1), "f"(x0));
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(r));
  }
  const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h));
  d0 = f.x;
  d1 = f.y;
  return r;
}

// Eight FP32 values -> kTerms 8-byte words of 8-bit values whose sum is the
// input up to the last term's rounding (each term takes the remainder left
// by the ones before it; the subtractions are exact).
template <bool kE5, int kTerms>
__device__ __forceinline__ void f8_terms(float *x, uint2 *out) {
#pragma unroll
  for (int t = 0; t < kTerms; ++t) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float d0, d1;
      w[i] = f8x2<kE5>(x[2 * i], x[2 * i + 1], d0, d1);
      x[2 * i] -= d0;
      x[2 * i + 1] -= d1;
    }
    out[t] = make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
  }
}

// Eight FP32 values -> F16 (round to nearest), then kTerms E5M2 terms of
// the F16 values.  E5M2 has F16's sign and exponent fields, so every E5M2
// value is an F16 value and the nearest E5M2 of an F16 (round to nearest,
// ties to even) leaves a remainder that F16 holds exactly: each term is the
// hardware conversion of the remainder so far, converted back and
// subtracted (an exact F16 subtraction).  Four terms of 3 significant bits
// hold all 11 bits of an F16.  (The inputs stay far below E5M2's largest
// finite value, so the saturating conversion never clips.)
template <int kTerms>
__device__ __forceinline__ void e5_terms_f16(const float *x, uint2 *out) {
  uint32_t h[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(h[i]) : "f"(x[2 * i + 1]), "f"(x[2 * i]));
#pragma unroll
  for (int t = 0; t < kTerms; ++t) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint16_t e;
      asm("cvt.rn.satfinite.e5m2x2.f16x2 %0, %1;" : "=h"(e) : "r"(h[i]));
      w[i] = e;
      if (t + 1 < kTerms) {
        uint32_t back;
        asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(back) : "h"(e));
        asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(h[i]) : "r"(h[i]), "r"(back));
      }
    }
    out[t] = make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
  }
}

// 2^e as a float, e in [-126, 127].
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((e + 127) << 23); }

// TMEM: this thread's lane, N consecutive 32-bit columns (N a multiple of 8),
// one wait for all of them.  The TMEM loads carry no memory clobber (TMEM is
// not memory the compiler tracks): volatile keeps them in order with the
// barrier waits and fences, and shared-memory traffic may overlap them.
template <int N>
__device__ __forceinline__ void tmem_load(uint32_t taddr, float *v) {
  static_assert(N % 8 == 0, "columns in groups of 8");
  uint32_t r[N];
#pragma unroll
  for (int c = 0; c < N; c += 8)
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=r"(r[c]), "=r"(r[c + 1]), "=r"(r[c + 2]), "=r"(r[c + 3]), "=r"(r[c + 4]),
          "=r"(r[c + 5]), "=r"(r[c + 6]), "=r"(r[c + 7])
        : "r"(taddr + c));
  asm volatile("tcgen05.wait::ld.sync.aligned;");
  // tie every register to the wait so no use is scheduled above it
#pragma unroll
  for (int c = 0; c < N; ++c) {
    asm volatile("" : "+r"(r[c]));
    v[c] = __uint_as_float(r[c]);
  }
}

// TMEM: this thread's lane, 8 columns from each of T blocks `stride`
// columns apart, summed in block order; one wait for all loads.
template <int T>
__device__ __forceinline__ void tmem_load_sum8(uint32_t taddr, int stride, float *v) {
  uint32_t r[T][8];
#pragma unroll
  for (int t = 0; t < T; ++t)
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=r"(r[t][0]), "=r"(r[t][1]), "=r"(r[t][2]), "=r"(r[t][3]), "=r"(r[t][4]),
          "=r"(r[t][5]), "=r"(r[t][6]), "=r"(r[t][7])
        : "r"(taddr + (uint32_t)(t * stride)));
  asm volatile("tcgen05.wait::ld.sync.aligned;");
#pragma unroll
  for (int t = 0; t < T; ++t)
#pragma unroll
    for (int c = 0; c < 8; ++c) asm volatile("" : "+r"(r[t][c]));
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float a = __uint_as_float(r[0][c]);
#pragma unroll
    for (int t = 1; t < T; ++t) a += __uint_as_float(r[t][c]);
    v[c] = a;
  }
}

// TMEM: this thread's lane, 4 columns from each of T blocks `stride`
// columns apart, summed in block order; one wait for all loads.
template <int T>
__device__ __forceinline__ void tmem_load_sum4(uint32_t taddr, int stride, float *v) {
  uint32_t r[T][4];
#pragma unroll
  for (int t = 0; t < T; ++t)
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[t][0]), "=r"(r[t][1]), "=r"(r[t][2]), "=r"(r[t][3])
                 : "r"(taddr + (uint32_t)(t * stride)));
  asm volatile("tcgen05.wait::ld.sync.aligned;");
#pragma unroll
  for (int t = 0; t < T; ++t)
#pragma unroll
    for (int c = 0; c < 4; ++c) asm volatile("" : "+r"(r[t][c]));
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    float a = __uint_as_float(r[0][c]);
#pragma unroll
    for (int t = 1; t < T; ++t) a += __uint_as_float(r[t][c]);
    v[c] = a;
  }
}

// TMEM: this thread's lane, C columns (a multiple of 4) from each of T
// blocks `stride` columns apart, summed in block order; every load is
// issued before the one wait.
template <int T, int C>
__device__ __forceinline__ void tmem_load_sum(uint32_t taddr, int stride, float *v) {
  static_assert(C % 4 == 0, "columns in groups of 4");
  uint32_t r[T][C];
#pragma unroll
  for (int t = 0; t < T; ++t)
#pragma unroll
    for (int c = 0; c < C; c += 4)
      asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(r[t][c]), "=r"(r[t][c + 1]), "=r"(r[t][c + 2]), "=r"(r[t][c + 3])
                   : "r"(taddr + (uint32_t)(t * stride + c)));
  asm volatile("tcgen05.wait::ld.sync.aligned;");
#pragma unroll
  for (int t = 0; t < T; ++t)
#pragma unroll
    for (int c = 0; c < C; ++c) asm volatile("" : "+r"(r[t][c]));
#pragma unroll
  for (int c = 0; c < C; ++c) {
    float a = __uint_as_float(r[0][c]);
#pragma unroll
    for (int t = 1; t < T; ++t) a += __uint_as_float(r[t][c]);
    v[c] = a;
  }
}

// TMEM: 4 columns of this thread's lane.
__device__ __forceinline__ void tmem_st4(uint32_t taddr, const float *v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr),
               "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
               "r"(__float_as_uint(v[3]))
               : "memory");
}

// Four FP32 values -> F16, then kTerms E5M2 terms of the F16 values (as
// e5_terms_f16, four values): out[t] holds term t of value i in byte i.
template <int kTerms>
__device__ __forceinline__ void e5_terms4(const float *x, uint32_t *out) {
  uint32_t h[2];
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(h[0]) : "f"(x[1]), "f"(x[0]));
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(h[1]) : "f"(x[3]), "f"(x[2]));
#pragma unroll
  for (int t = 0; t < kTerms; ++t) {
    uint32_t w[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      uint16_t e;
      asm("cvt.rn.satfinite.e5m2x2.f16x2 %0, %1;" : "=h"(e) : "r"(h[i]));
      w[i] = e;
      if (t + 1 < kTerms) {
        uint32_t back;
        asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(back) : "h"(e));
        asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(h[i]) : "r"(h[i]), "r"(back));
      }
    }
    out[t] = w[0] | (w[1] << 16);
  }
}

// Sum (kMax: maximum) of four per-lane values over the 32 lanes of a warp,
// by a fixed butterfly (halving the values each lane keeps, then full
// reductions): every lane returns the warp result of value (lane >> 3) & 3.
template <bool kMax>
__device__ __forceinline__ float warp_reduce4(const float *e, int lane) {
  auto op = [](float a, float b) { return kMax ? fmaxf(a, b) : a + b; };
  const bool b4 = lane & 16, b3 = lane & 8;
  float w2[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float keep = b4 ? e[2 + i] : e[i], give = b4 ? e[i] : e[2 + i];
    w2[i] = op(keep, __shfl_xor_sync(0xffffffffu, give, 16));
  }
  float x = op(b3 ? w2[1] : w2[0], __shfl_xor_sync(0xffffffffu, b3 ? w2[0] : w2[1], 8));
  x = op(x, __shfl_xor_sync(0xffffffffu, x, 4));
  x = op(x, __shfl_xor_sync(0xffffffffu, x, 2));
  x = op(x, __shfl_xor_sync(0xffffffffu, x, 1));
  return x;
}

}  // namespace lse_ptx
