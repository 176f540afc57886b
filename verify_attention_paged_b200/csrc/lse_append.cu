// K/V append: the new tokens of a decode or verify step written into their
// fragments through the page tables (LSE releases, v0.4.20 "K/V memory
// management and automatic split attention"), cast from FP32 to the storage
// format.
//
// One warp per (new token, kv head): each lane loads a contiguous D/32
// slice of the head's K and V vectors, the warp finds the token's sequence
// by a 32-way search over new_offsets and the fragment through the page
// table, and each lane stores its converted slices (coalesced across the
// warp).  Casts: nearest value, ties to
// even (cvt.rn); FP8 through cvt.rn.satfinite (saturating at the largest
// finite value); F16 and BF16 overflow to infinity.  With per-vector scales
// (8-bit arenas) the warp also takes each vector's largest magnitude (a
// butterfly max), its scale = that / the format's largest finite value (1
// for a zero vector), stores the elements divided by it (FP32 division,
// correctly rounded) and lane 0 writes the scale to the [kv_head][token]
// block of the fragment.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "lse_internal.h"

namespace {

constexpr int kWarpsPerBlock = 8;

// Two FP32 values -> the storage format's bits, x0 in the low half.
template <int DT>
__device__ __forceinline__ uint32_t pack2(float x0, float x1);
template <>
__device__ __forceinline__ uint32_t pack2<LSE_KV_F16>(float x0, float x1) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(x1), "f"(x0));
  return r;
}
template <>
__device__ __forceinline__ uint32_t pack2<LSE_KV_BF16>(float x0, float x1) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(x1), "f"(x0));
  return r;
}
template <>
__device__ __forceinline__ uint32_t pack2<LSE_KV_FP8_E4M3>(float x0, float x1) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(x1), "f"(x0));
  return r;
}
template <>
__device__ __forceinline__ uint32_t pack2<LSE_KV_FP8_E5M2>(float x0, float x1) {
  uint16_t r;
  asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(x1), "f"(x0));
  return r;
}

// This lane's kPer consecutive FP32 elements (already loaded) -> stored
// bytes at dst.
template <int DT, int kPer>
__device__ __forceinline__ void store_slice(const float *x, uint8_t *dst) {
  if constexpr (DT == LSE_KV_F32) {
#pragma unroll
    for (int k = 0; k < kPer; k += 2)
      *reinterpret_cast<float2 *>(dst + 4 * k) = make_float2(x[k], x[k + 1]);
  } else if constexpr (DT == LSE_KV_F16 || DT == LSE_KV_BF16) {
#pragma unroll
    for (int k = 0; k < kPer; k += 2)
      *reinterpret_cast<uint32_t *>(dst + 2 * k) = pack2<DT>(x[k], x[k + 1]);
  } else {
    // FP8: pairs of bytes
#pragma unroll
    for (int k = 0; k < kPer; k += 2)
      *reinterpret_cast<uint16_t *>(dst + k) = (uint16_t)pack2<DT>(x[k], x[k + 1]);
  }
}

template <int DT, int D>
__global__ void __launch_bounds__(kWarpsPerBlock * 32) kv_append_kernel(const AppendParams a) {
  constexpr int kPer = D / 32;
  constexpr int kEs = DT == LSE_KV_F32 ? 4 : (DT == LSE_KV_F16 || DT == LSE_KV_BF16) ? 2 : 1;
  const int lane = threadIdx.x & 31;
  const long long v = (long long)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  if (v >= (long long)a.total_new * a.n_kv_heads) return;  // uniform per warp
  const int i = (int)(v / a.n_kv_heads), g = (int)(v - (long long)i * a.n_kv_heads);
  // the lane's slices of K and V first: their address does not depend on
  // the sequence, so the loads overlap the search below
  const long long src = ((long long)i * a.n_kv_heads + g) * D + lane * kPer;
  float xk[kPer], xv[kPer];
#pragma unroll
  for (int k = 0; k < kPer; k += 2) {
    const float2 fk = *reinterpret_cast<const float2 *>(a.k_new + src + k);
    const float2 fv = *reinterpret_cast<const float2 *>(a.v_new + src + k);
    xk[k] = fk.x;
    xk[k + 1] = fk.y;
    xv[k] = fv.x;
    xv[k + 1] = fv.y;
  }
  float sk = 1.f, sv = 1.f;
  if constexpr (DT == LSE_KV_FP8_E4M3 || DT == LSE_KV_FP8_E5M2) {
    if (a.scales) {
      float mk = 0.f, mv = 0.f;
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        mk = fmaxf(mk, fabsf(xk[k]));
        mv = fmaxf(mv, fabsf(xv[k]));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        mk = fmaxf(mk, __shfl_xor_sync(0xffffffffu, mk, o));
        mv = fmaxf(mv, __shfl_xor_sync(0xffffffffu, mv, o));
      }
      constexpr float kFmtMax = DT == LSE_KV_FP8_E4M3 ? 448.f : 57344.f;
      if (mk > 0.f) sk = __fdiv_rn(mk, kFmtMax);
      if (mv > 0.f) sv = __fdiv_rn(mv, kFmtMax);
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        xk[k] = __fdiv_rn(xk[k], sk);
        xv[k] = __fdiv_rn(xv[k], sv);
      }
    }
  }
  // the token's sequence, the last s with new_offsets[s] <= i: each round the
  // 32 lanes test 32 evenly spaced offsets of the remaining range
  int lo = 0, span = a.n_seqs;  // s in [lo, lo + span)
  while (span > 1) {
    const int step = (span + 31) / 32;
    const int idx = lo + lane * step;
    const bool le = idx < lo + span && a.new_offsets[idx] <= i;
    const unsigned m = __ballot_sync(0xffffffffu, le);
    const int top = m ? 31 - __clz(m) : 0;  // the last lane whose offset is <= i
    lo += top * step;
    span = min(step, span - top * step);
  }
  const int s = lo;
  const int first = a.new_offsets[s];
  if (first > i || i >= a.new_offsets[s + 1]) {
    if (lane == 0 && a.err) atomicOr(a.err, LSE_DEVERR_BAD_LENGTH);
    return;
  }
  const long long pos = (long long)a.seq_lens_before[s] + (i - first);
  const long long page = pos / a.tokens_per_fragment;
  const long long slot = pos - page * a.tokens_per_fragment;
#pragma unroll
  for (int kv = 0; kv < 2; ++kv) {
    const int32_t *table = kv ? a.v_pages : a.k_pages;
    int frag = -1;
    if (pos >= 0 && page < a.max_pages) frag = table[(long long)s * a.max_pages + page];
    if (frag < 0 || frag >= a.n_fragments) {
      if (lane == 0 && a.err) atomicOr(a.err, LSE_DEVERR_BAD_FRAGMENT);
      continue;
    }
    const int c = frag / a.frags_per_chunk;
    uint8_t *dst = reinterpret_cast<uint8_t *>(a.chunk_base[c]) +
                   (long long)(frag - c * a.frags_per_chunk) * a.fragment_bytes +
                   ((slot * a.n_kv_heads + g) * D + lane * kPer) * kEs;
    store_slice<DT, kPer>(kv ? xv : xk, dst);
    if (a.scales && lane == 0)
      a.scales[((long long)frag * a.n_kv_heads + g) * a.tokens_per_fragment + slot] = kv ? sv : sk;
  }
}

template <int DT>
int launch_dt(const AppendParams &a, int D, cudaStream_t st) {
  const long long vecs = (long long)a.total_new * a.n_kv_heads;
  const unsigned blocks = (unsigned)((vecs + kWarpsPerBlock - 1) / kWarpsPerBlock);
  switch (D) {
    case 64: kv_append_kernel<DT, 64><<<blocks, kWarpsPerBlock * 32, 0, st>>>(a); break;
    case 128: kv_append_kernel<DT, 128><<<blocks, kWarpsPerBlock * 32, 0, st>>>(a); break;
    case 256: kv_append_kernel<DT, 256><<<blocks, kWarpsPerBlock * 32, 0, st>>>(a); break;
    default: return (int)cudaErrorInvalidValue;
  }
  return (int)cudaGetLastError();
}

}  // namespace

int lse_launch_kv_append(const AppendParams &a, int dtype, int head_dim, void *stream) {
  if (a.total_new <= 0) return 0;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  switch (dtype) {
    case LSE_KV_F32: return launch_dt<LSE_KV_F32>(a, head_dim, st);
    case LSE_KV_F16: return launch_dt<LSE_KV_F16>(a, head_dim, st);
    case LSE_KV_BF16: return launch_dt<LSE_KV_BF16>(a, head_dim, st);
    case LSE_KV_FP8_E4M3: return launch_dt<LSE_KV_FP8_E4M3>(a, head_dim, st);
    case LSE_KV_FP8_E5M2: return launch_dt<LSE_KV_FP8_E5M2>(a, head_dim, st);
  }
  return (int)cudaErrorInvalidValue;
}
