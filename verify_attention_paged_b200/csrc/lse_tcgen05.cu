// Tensor-core (tcgen05) partial pass of split-KV paged attention, sm_100a.
//
// What it computes is the partial pass of the split attention described on
// the LSE releases page (v0.4.19 "Long-context split attention": one
// partial family whose verifier rows share K/V loads; v0.4.21: K/V reads
// shared across query heads and token rows; v0.4.20: partitions sized from
// the K/V table capacity, empty partitions skipped).  How it computes it is
// B200-specific:
//
//  * Persistent grid, one CTA per SM.  The live key tiles of every
//    (sequence, kv head) segment are laid end to end and cut into one
//    contiguous, equal, non-empty range per working CTA (min(grid, tiles)
//    of them), so every SM streams the same number of bytes.  A CTA writes one partial result per segment piece it covers;
//    pieces of a segment are numbered by CTA, so the merge knows which
//    workspace slots are live without any host round trip.  Capacity that
//    holds no live key is never enumerated (the empty partitions are
//    skipped).
//  * K/V tiles of 128 keys x 128 dims of one kv head are brought into shared
//    memory by TMA (cp.async.bulk.tensor, 128-byte swizzle, no multicast)
//    straight out of the fragments through the page table, in a multi-stage
//    mbarrier pipeline, and each tile is read once for all (row, head) pairs.
//  * Scores are computed transposed, S^T = K Q^T (M = 128 keys, N = pairs),
//    so the tile's keys fill the 128-row MMA whatever the number of query
//    rows; the output is O^T = V^T P^T (M = 128 dims).  Both accumulate in
//    TMEM in FP32.  Q and P carry a hi + lo pair of 16-bit terms (one term
//    holds the value rounded to the storage's 16-bit format, the other the
//    rounding error) so the products keep ~16 mantissa bits and only the
//    K/V storage rounding remains.
//  * Softmax: one thread per key reads its row of S from TMEM.  The running
//    maximum is rescaled lazily: only when a score exceeds it by more than
//    2^8 are the maxima recomputed and the TMEM output rescaled.
//
// Roles (256 threads): warp 0 TMA producer, warp 1 MMA issuer (and TMEM
// owner), warps 2-3 stage Q, warps 4-7 softmax and epilogue.  Every wait is
// bounded: a wait that runs out sets LSE_DEVERR_TIMEOUT and every role
// leaves its loop; TMEM is released and outstanding copies are drained
// before the CTA exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "lse_internal.h"

namespace {

constexpr int kTK = 128;           // keys per tile = M of the score product
constexpr int kD = 128;            // head dim = M of the output product
constexpr int kThreads = 256;
constexpr float kTau = 8.f;        // lazy-rescale threshold (log2 units)
constexpr long long kWaitCycles = 4000000000ll;  // ~2 s at 2 GHz
constexpr int kRegionBytes = kTK * 128;          // 128 rows x 128 B (64 dims)
constexpr int kStageBytes = 4 * kRegionBytes;    // K (2 regions) + V (2 regions)

struct __align__(64) TcParams {
  CUtensorMap maps[LSE_MAX_TMA_CHUNKS];
  LseKernelParams p;
  int n_ctas;
  int n_slots;
  int stages;
  int box_tokens;
};

// ---- PTX helpers --------------------------------------------------------------

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

// Wait for the phase of `bar` with the given parity; false when the wait ran
// out (then the CTA-wide abort flag is set) or another role aborted.
__device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                       unsigned int *err) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 31u) == 0) {
      if (*abort_flag) return false;
      if (clock64() - t0 > kWaitCycles) {
        *abort_flag = 1;
        atomicOr(err, LSE_DEVERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Time-bounded wait that ignores the abort flag: used to drain copies and
// MMAs already in flight before the CTA releases TMEM and exits.
__device__ __noinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
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

// UMMA shared-memory matrix descriptor.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
}
constexpr uint32_t kLayoutNone = 0;
constexpr uint32_t kLayoutSw128 = 2;

// Instruction descriptor, kind::f16, FP32 accumulation.
__host__ __device__ constexpr uint32_t instr_desc(uint32_t ab_fmt, uint32_t a_mn, uint32_t b_mn,
                                                  uint32_t M, uint32_t N) {
  return (1u << 4) | (ab_fmt << 7) | (ab_fmt << 10) | (a_mn << 15) | (b_mn << 16) |
         ((N >> 3) << 17) | ((M >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// 8 consecutive TMEM columns of this thread's lane; the wait is tied to the
// destination registers so no use can be hoisted above it.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float *v) {
  uint32_t r[8];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7])
               :
               : "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
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

// Round an FP32 value to the 16-bit operand format: the nearest value plus
// the rounding error in the same format (hi + lo carries ~16 mantissa bits).
template <int DT>
struct Op16;
template <>
struct Op16<LSE_KV_BF16> {
  static constexpr uint32_t kFmt = 1;
  static __device__ __forceinline__ void split(float x, uint16_t &hi, uint16_t &lo) {
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    const __nv_bfloat16 l = __float2bfloat16_rn(x - __bfloat162float(h));
    hi = *reinterpret_cast<const uint16_t *>(&h);
    lo = *reinterpret_cast<const uint16_t *>(&l);
  }
};
template <>
struct Op16<LSE_KV_F16> {
  static constexpr uint32_t kFmt = 0;
  static __device__ __forceinline__ void split(float x, uint16_t &hi, uint16_t &lo) {
    const __half h = __float2half_rn(x);
    const __half l = __float2half_rn(x - __half2float(h));
    hi = *reinterpret_cast<const uint16_t *>(&h);
    lo = *reinterpret_cast<const uint16_t *>(&l);
  }
};

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// ---- work decomposition ---------------------------------------------------------

// Number of 128-key tiles of sequence s (0 for idle or malformed sequences).
__device__ __forceinline__ int seq_tiles(const LseKernelParams &p, int s, int &L, int &row0,
                                         int &R) {
  L = p.seq_lens[s];
  row0 = p.row_offsets[s];
  R = p.row_offsets[s + 1] - row0;
  const long long cap = (long long)p.max_pages * p.tokens_per_fragment;
  if (row0 < 0 || R < 0 || R > p.max_rows || row0 + R > p.max_total_rows || R > L ||
      (long long)L > cap)
    return -1;
  return R == 0 ? 0 : (L + kTK - 1) / kTK;
}

// Walks the CTA's contiguous range of global tiles, segment by segment.
struct TileIter {
  int s, g, tile, n_tiles;   // segment (sequence, kv head) and tile within it
  int L, row0, R;
  long long seg_first;       // global index of the segment's first tile
  long long t, t_end;        // current / end global tile

  __device__ void next_seq(const LseKernelParams &p) {
    // advance to the next sequence with tiles, starting at s
    while (s < p.n_seqs) {
      const int n = seq_tiles(p, s, L, row0, R);
      if (n > 0) {
        n_tiles = n;
        return;
      }
      ++s;
    }
  }
  __device__ void init(const LseKernelParams &p, long long t_begin, long long t_stop) {
    t = t_begin;
    t_end = t_stop;
    s = 0;
    long long base = 0;
    n_tiles = 0;
    if (t >= t_end) return;
    next_seq(p);
    while (base + (long long)p.n_kv_heads * n_tiles <= t) {
      base += (long long)p.n_kv_heads * n_tiles;
      ++s;
      next_seq(p);
    }
    g = int((t - base) / n_tiles);
    tile = int((t - base) - (long long)g * n_tiles);
    seg_first = base + (long long)g * n_tiles;
  }
  __device__ bool valid() const { return t < t_end; }
  __device__ bool seg_start(long long t_begin) const { return t == t_begin || tile == 0; }
  __device__ bool seg_end() const { return t == t_end - 1 || tile == n_tiles - 1; }
  __device__ void advance(const LseKernelParams &p) {
    ++t;
    if (t >= t_end) return;
    if (++tile == n_tiles) {
      tile = 0;
      seg_first += n_tiles;
      if (++g == p.n_kv_heads) {
        g = 0;
        ++s;
        next_seq(p);
      }
    }
  }
};

// CTA whose range holds global tile t, for ranges [c U / C, (c+1) U / C).
__device__ __forceinline__ int cta_of_tile(long long t, long long U, int C) {
  return int(((t + 1) * (long long)C - 1) / U);
}

// ---- shared-memory layout --------------------------------------------------------

template <int P8>
struct TcLayout {
  static constexpr int kN = 2 * P8;                  // hi + lo columns
  static constexpr int kQRegion = kN * 128;          // one 64-dim region of Q rows
  static constexpr int kQBytes = 2 * kQRegion;
  static constexpr int kPLbo = (kN / 8) * 128;       // P: stride between 8-key groups
  static constexpr int kPBytes = kTK * kN * 2;
  static constexpr int kTmemCols = (3 * kN <= 64) ? 64 : (3 * kN <= 128) ? 128
                                 : (3 * kN <= 256) ? 256 : 512;
  // misc block
  static constexpr int kBars = 24;
  static constexpr int kMiscBytes = kBars * 8 + 16 + 64 * 4 * 2 + 4 * 64 * 4 + 64 * 8 + 64 * 4;
  static int smem_bytes(int stages) {
    return 1024 + stages * kStageBytes + 2 * kQBytes + kPBytes + kMiscBytes;
  }
};

// barrier indices in the misc block
enum {
  kBarFull = 0,    // [4]
  kBarEmpty = 4,   // [4]
  kBarSFull = 8,
  kBarPFull = 9,
  kBarQFull = 10,  // [2]
  kBarQEmpty = 12, // [2]
  kBarOFull = 14,  // [2]
  kBarOEmpty = 16, // [2]
  kBarDone = 18,
};

template <int DT, int P8>
__global__ void __launch_bounds__(kThreads, 1)
    partial_tcgen05_kernel(const __grid_constant__ TcParams tp) {
  using Lay = TcLayout<P8>;
  using Op = Op16<DT>;
  constexpr int kN = Lay::kN;
  const LseKernelParams &p = tp.p;
  const int NS = tp.stages;
  const int cta = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t stage_base = sbase;
  const uint32_t q_base = sbase + NS * kStageBytes;
  const uint32_t p_base = q_base + 2 * Lay::kQBytes;
  uint8_t *misc = smem + NS * kStageBytes + 2 * Lay::kQBytes + Lay::kPBytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(misc);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + Lay::kBars * 8);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + Lay::kBars * 8 + 4);
  long long *shared_u = reinterpret_cast<long long *>(misc + Lay::kBars * 8 + 8);
  float *m_run = reinterpret_cast<float *>(misc + Lay::kBars * 8 + 16);  // [64]
  float *alpha = m_run + 64;                                             // [64]
  float *red = alpha + 64;                                               // [4][64]
  unsigned long long *masks = reinterpret_cast<unsigned long long *>(red + 4 * 64);  // [64]
  int *pair_row = reinterpret_cast<int *>(masks + 64);                   // [64]
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  // ---- prologue: total live tiles, barriers, TMEM -------------------------------
  if (tid == 0) {
    long long U = 0;
    bool bad = false;
    for (int s = 0; s < p.n_seqs; ++s) {
      int L, r0, R;
      const int n = seq_tiles(p, s, L, r0, R);
      if (n < 0) bad = true;
      else U += n;
    }
    if (bad && cta == 0) atomicOr(p.err, LSE_DEVERR_BAD_LENGTH);
    *shared_u = U * p.n_kv_heads;
    *abort_flag = 0;
    for (int i = 0; i < 4; ++i) {
      mbar_init(bar(kBarFull + i), 1);
      mbar_init(bar(kBarEmpty + i), 1);
    }
    mbar_init(bar(kBarSFull), 1);
    mbar_init(bar(kBarPFull), 128);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kBarQFull + i), 64);
      mbar_init(bar(kBarQEmpty + i), 1);
      mbar_init(bar(kBarOFull + i), 1);
      mbar_init(bar(kBarOEmpty + i), 128);
    }
    mbar_init(bar(kBarDone), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (tid < 64) pair_row[tid] = tid / p.group;
  __syncthreads();
  const long long U = *shared_u;
  // working CTAs: never more than tiles, so no working range is empty and a
  // segment's pieces never outnumber its tiles
  const int C = (int)(U < tp.n_ctas ? U : tp.n_ctas);
  if (cta >= C) return;  // nothing for this CTA (uniform)
  const long long t_begin = U * cta / C, t_stop = U * (cta + 1) / C;

  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(Lay::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_s = tmem;                 // S^T: lanes = keys, cols [0, N)
  auto tmem_o = [&](int slot) { return tmem + (uint32_t)(kN * (1 + slot)); };

  const int T = p.tokens_per_fragment;
  const int box_t = tp.box_tokens;
  const int G = p.group;

  if (warp == 0) {
    // ============================ TMA producer ============================
    if (lane == 0) {
      TileIter it;
      it.init(p, t_begin, t_stop);
      int n = 0;
      for (; it.valid(); it.advance(p), ++n) {
        const int st = n % NS;
        if (!mbar_wait(bar(kBarEmpty + st), ((n / NS) & 1) ^ 1, abort_flag, p.err)) break;
        const int key0 = it.tile * kTK;
        const int nbox = box_t >= kTK ? 1 : kTK / box_t;
        // which boxes exist (live and naming a fragment), K and V separately
        uint32_t kmask = 0, vmask = 0;
        for (int b = 0; b < nbox; ++b) {
          const int kb = key0 + b * box_t;
          if (kb >= it.L) break;
          const long long e = (long long)it.s * p.max_pages + kb / T;
          const int fk = p.k_pages[e], fv = p.v_pages[e];
          if (fk >= 0 && fk < p.n_fragments) kmask |= 1u << b;
          else atomicOr(p.err, LSE_DEVERR_BAD_FRAGMENT);
          if (fv >= 0 && fv < p.n_fragments) vmask |= 1u << b;
          else atomicOr(p.err, LSE_DEVERR_BAD_FRAGMENT);
        }
        const uint32_t bytes =
            (uint32_t)(__popc(kmask) + __popc(vmask)) * 2u * (uint32_t)box_t * 128u;
        const uint32_t fb = bar(kBarFull + st);
        mbar_expect_tx(fb, bytes);
        const uint32_t kdst = stage_base + st * kStageBytes;
        const uint32_t vdst = kdst + 2 * kRegionBytes;
        for (int b = 0; b < nbox; ++b) {
          const int kb = key0 + b * box_t;
          const long long e = (long long)it.s * p.max_pages + kb / T;
          const int off = kb % T;
          if (kmask >> b & 1u) {
            const int f = p.k_pages[e];
            const int c = f / p.frags_per_chunk;
            const int z = (f - c * p.frags_per_chunk) * T + off;
            for (int h = 0; h < 2; ++h)
              tma_load_3d(kdst + h * kRegionBytes + b * box_t * 128, &tp.maps[c], fb, 0,
                          it.g * 2 + h, z);
          }
          if (vmask >> b & 1u) {
            const int f = p.v_pages[e];
            const int c = f / p.frags_per_chunk;
            const int z = (f - c * p.frags_per_chunk) * T + off;
            for (int h = 0; h < 2; ++h)
              tma_load_3d(vdst + h * kRegionBytes + b * box_t * 128, &tp.maps[c], fb, 0,
                          it.g * 2 + h, z);
          }
        }
      }
      // drain: every stage issued must have landed before the CTA exits
      for (int k = (n > NS ? n - NS : 0); k < n; ++k) mbar_drain(bar(kBarFull + k % NS), (k / NS) & 1);
    }
  } else if (warp == 1) {
    // ============================ MMA issuer ==============================
    if (lane == 0) {
      constexpr uint32_t idesc_qk = instr_desc(Op::kFmt, 0, 0, kTK, kN);
      constexpr uint32_t idesc_pv = instr_desc(Op::kFmt, 1, 1, kD, kN);
      TileIter it;
      it.init(p, t_begin, t_stop);
      int n = 0, seg = -1;
      for (; it.valid(); it.advance(p), ++n) {
        const bool first = it.seg_start(t_begin), last = it.seg_end();
        if (first) {
          ++seg;
          if (!mbar_wait(bar(kBarQFull + (seg & 1)), (seg >> 1) & 1, abort_flag, p.err)) break;
          if (!mbar_wait(bar(kBarOEmpty + (seg & 1)), ((seg >> 1) & 1) ^ 1, abort_flag, p.err))
            break;
        }
        const int st = n % NS;
        if (!mbar_wait(bar(kBarFull + st), (n / NS) & 1, abort_flag, p.err)) break;
        tc_fence_after();
        const uint32_t kaddr = stage_base + st * kStageBytes;
        const uint32_t vaddr = kaddr + 2 * kRegionBytes;
        const uint32_t qaddr = q_base + (seg & 1) * Lay::kQBytes;
        // S^T = K Q^T : 8 steps of 16 dims
#pragma unroll
        for (int k = 0; k < kD / 16; ++k) {
          const uint64_t a = smem_desc(kaddr + (k >> 2) * kRegionBytes + (k & 3) * 32, 16, 1024,
                                       kLayoutSw128);
          const uint64_t b = smem_desc(qaddr + (k >> 2) * Lay::kQRegion + (k & 3) * 32, 16,
                                       1024, kLayoutSw128);
          mma_f16(tmem_s, a, b, idesc_qk, k > 0);
        }
        mma_commit(bar(kBarSFull));
        if (last) mma_commit(bar(kBarQEmpty + (seg & 1)));
        if (!mbar_wait(bar(kBarPFull), n & 1, abort_flag, p.err)) break;
        tc_fence_after();
        // O^T (+)= V^T P^T : 8 steps of 16 keys
#pragma unroll
        for (int k = 0; k < kTK / 16; ++k) {
          const uint64_t a =
              smem_desc(vaddr + k * 2048, kRegionBytes, 1024, kLayoutSw128);  // MN-major
          const uint64_t b =
              smem_desc(p_base + k * 2 * Lay::kPLbo, Lay::kPLbo, 128, kLayoutNone);  // MN-major
          mma_f16(tmem_o(seg & 1), a, b, idesc_pv, (!first || k > 0) ? 1u : 0u);
        }
        mma_commit(bar(kBarEmpty + st));
        if (last) mma_commit(bar(kBarOFull + (seg & 1)));
      }
      // every MMA issued has completed before TMEM is released
      mma_commit(bar(kBarDone));
      mbar_drain(bar(kBarDone), 0);
    }
  } else if (warp < 4) {
    // ============================ Q staging ===============================
    const int qt = tid - 64;  // 0..63
    TileIter it;
    it.init(p, t_begin, t_stop);
    int seg = -1;
    for (; it.valid(); it.advance(p)) {
      if (!it.seg_start(t_begin)) continue;
      ++seg;
      const int slot = seg & 1;
      if (!mbar_wait(bar(kBarQEmpty + slot), ((seg >> 1) & 1) ^ 1, abort_flag, p.err)) break;
      uint8_t *qs = smem + (q_base - sbase) + slot * Lay::kQBytes;
      const int P = G * it.R;
      // row n < P8 holds hi of pair n, row P8 + n its lo; 16 chunks of 8 dims
      for (int item = qt; item < P8 * 16; item += 64) {
        const int n = item >> 4, c = item & 15;
        float x[8];
        if (n < P) {
          const int r = n / G, h = it.g * G + (n - r * G);
          const float4 *src = reinterpret_cast<const float4 *>(
              p.q + ((long long)(it.row0 + r) * p.n_q_heads + h) * kD + c * 8);
          const float4 a = __ldg(src), b2 = __ldg(src + 1);
          x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
          x[4] = b2.x; x[5] = b2.y; x[6] = b2.z; x[7] = b2.w;
#pragma unroll
          for (int i = 0; i < 8; ++i) x[i] *= p.scale_log2;
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) x[i] = 0.f;
        }
        uint16_t hi[8], lo[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) Op::split(x[i], hi[i], lo[i]);
        const int region = c >> 3, cc = c & 7;
        const uint32_t rh = n, rl = P8 + n;
        const uint32_t ohi = region * Lay::kQRegion + (rh >> 3) * 1024 + (rh & 7) * 128 +
                             ((cc ^ (rh & 7)) << 4);
        const uint32_t olo = region * Lay::kQRegion + (rl >> 3) * 1024 + (rl & 7) * 128 +
                             ((cc ^ (rl & 7)) << 4);
        uint4 vh, vl;
        vh.x = hi[0] | (uint32_t)hi[1] << 16; vh.y = hi[2] | (uint32_t)hi[3] << 16;
        vh.z = hi[4] | (uint32_t)hi[5] << 16; vh.w = hi[6] | (uint32_t)hi[7] << 16;
        vl.x = lo[0] | (uint32_t)lo[1] << 16; vl.y = lo[2] | (uint32_t)lo[3] << 16;
        vl.z = lo[4] | (uint32_t)lo[5] << 16; vl.w = lo[6] | (uint32_t)lo[7] << 16;
        *reinterpret_cast<uint4 *>(qs + ohi) = vh;
        *reinterpret_cast<uint4 *>(qs + olo) = vl;
      }
      fence_proxy_async();
      mbar_arrive(bar(kBarQFull + slot));
    }
  } else {
    // ===================== softmax and epilogue (128 threads) =====================
    const int j = tid - 128;          // key within tile = TMEM lane (scores)
    const int quarter = warp - 4;     // TMEM lane quarter of this warp
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    TileIter it;
    it.init(p, t_begin, t_stop);
    int n = 0, seg = -1;
    float l[P8];
    bool ok = true;
    for (; it.valid() && ok; it.advance(p), ++n) {
      const bool first = it.seg_start(t_begin), last = it.seg_end();
      const int P = G * it.R;
      const int Cctx = it.L - it.R;
      if (first) {
        ++seg;
        if (j < P8) m_run[j] = -INFINITY;
        if (j < it.R)
          masks[j] = p.row_masks ? p.row_masks[it.row0 + j]
                                 : (j >= 63 ? ~0ull : ((1ull << (j + 1)) - 1ull));
#pragma unroll
        for (int q = 0; q < P8; ++q) l[q] = 0.f;
        named_sync(1, 128);
      }
      if (!mbar_wait(bar(kBarSFull), n & 1, abort_flag, p.err)) { ok = false; break; }
      tc_fence_after();
      __syncwarp();
      // scores of key j for every pair: hi + lo columns
      float s[P8];
#pragma unroll
      for (int c = 0; c < P8; c += 8) {
        float hi[8], lo[8];
        tmem_ld8(tmem_s + lane_off + c, hi);
        tmem_ld8(tmem_s + lane_off + P8 + c, lo);
#pragma unroll
        for (int i = 0; i < 8; ++i) s[c + i] = hi[i] + lo[i];
      }
      const int key = it.tile * kTK + j;
      bool kvalid = key < it.L;
      if (kvalid) {
        const long long e = (long long)it.s * p.max_pages + key / T;
        const int fk = p.k_pages[e], fv = p.v_pages[e];
        kvalid = fk >= 0 && fk < p.n_fragments && fv >= 0 && fv < p.n_fragments;
      }
#pragma unroll
      for (int q = 0; q < P8; ++q) {
        bool vis = kvalid && q < P;
        if (vis && key >= Cctx) vis = (masks[pair_row[q]] >> (key - Cctx)) & 1ull;
        if (!vis) s[q] = -INFINITY;
      }
      // lazy maximum: rescale only when some score passes the running max by 2^tau
      bool need = false;
#pragma unroll
      for (int q = 0; q < P8; ++q) need |= s[q] > m_run[q] + kTau;
      if (named_or(1, 128, need)) {
#pragma unroll
        for (int q = 0; q < P8; ++q) {
          const float v = warp_max(s[q]);
          if (lane == 0) red[quarter * 64 + q] = v;
        }
        named_sync(1, 128);
        if (j < P8) {
          const float mo = m_run[j];
          const float mt = fmaxf(fmaxf(red[j], red[64 + j]), fmaxf(red[128 + j], red[192 + j]));
          const float mn = fmaxf(mo, mt);
          alpha[j] = (mn == -INFINITY) ? 1.f : exp2f(mo - mn);
          m_run[j] = mn;
        }
        named_sync(1, 128);
#pragma unroll
        for (int q = 0; q < P8; ++q) l[q] *= alpha[q];
        if (!first) {
          __syncwarp();
          // the previous tile's P.V has completed (the score commit covers it)
          const uint32_t ob = tmem_o(seg & 1) + lane_off;
#pragma unroll
          for (int c = 0; c < P8; c += 8) {
            float v[8], w[8];
            tmem_ld8(ob + c, v);
            tmem_ld8(ob + P8 + c, w);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              v[i] *= alpha[c + i];
              w[i] *= alpha[c + i];
            }
            tmem_st8(ob + c, v);
            tmem_st8(ob + P8 + c, w);
          }
          tmem_st_wait();
        }
      }
      // probabilities (hi + lo operand terms) into the P buffer, row j
      uint8_t *prow = smem + (p_base - sbase) + (j >> 3) * Lay::kPLbo + (j & 7) * 16;
#pragma unroll
      for (int c = 0; c < P8; c += 8) {
        uint16_t hi[8], lo[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float x = s[c + i];
          const float e = (x == -INFINITY) ? 0.f : exp2f(x - m_run[c + i]);
          l[c + i] += e;
          Op::split(e, hi[i], lo[i]);
        }
        uint4 vh, vl;
        vh.x = hi[0] | (uint32_t)hi[1] << 16; vh.y = hi[2] | (uint32_t)hi[3] << 16;
        vh.z = hi[4] | (uint32_t)hi[5] << 16; vh.w = hi[6] | (uint32_t)hi[7] << 16;
        vl.x = lo[0] | (uint32_t)lo[1] << 16; vl.y = lo[2] | (uint32_t)lo[3] << 16;
        vl.z = lo[4] | (uint32_t)lo[5] << 16; vl.w = lo[6] | (uint32_t)lo[7] << 16;
        *reinterpret_cast<uint4 *>(prow + (c >> 3) * 128) = vh;
        *reinterpret_cast<uint4 *>(prow + ((P8 + c) >> 3) * 128) = vl;
      }
      if (!kvalid) {
        // a dead slot may hold any bits: give it a zero V row (P is 0 there)
        const int st = n % NS;
        mbar_wait(bar(kBarFull + st), (n / NS) & 1, abort_flag, p.err);
        uint8_t *v0 = smem + st * kStageBytes + 2 * kRegionBytes + j * 128;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4 *>(v0 + h * kRegionBytes + c * 16) = make_uint4(0, 0, 0, 0);
      }
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(bar(kBarPFull));

      if (last) {
        // ---- epilogue: normalised partial output and its log2-sum-exp ----
#pragma unroll
        for (int q = 0; q < P8; ++q) {
          const float v = warp_sum(l[q]);
          if (lane == 0) red[quarter * 64 + q] = v;
        }
        named_sync(1, 128);
        if (!mbar_wait(bar(kBarOFull + (seg & 1)), (seg >> 1) & 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        __syncwarp();
        const int c_first = cta_of_tile(it.seg_first, U, C);
        const int slot = cta - c_first;
        const int d = j;  // output lane = head dim
        const uint32_t ob = tmem_o(seg & 1) + lane_off;
#pragma unroll
        for (int c = 0; c < P8; c += 8) {
          float v[8], w[8];
          tmem_ld8(ob + c, v);
          tmem_ld8(ob + P8 + c, w);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int q = c + i;
            if (q < P) {
              const float lt = red[q] + red[64 + q] + red[128 + q] + red[192 + q];
              const int r = pair_row[q], h = it.g * G + (q - r * G);
              const long long idx =
                  ((long long)(it.row0 + r) * p.n_q_heads + h) * tp.n_slots + slot;
              p.o_part[idx * kD + d] = lt > 0.f ? (v[i] + w[i]) / lt : 0.f;
              if (d == q) p.lse_part[idx] = lt > 0.f ? m_run[q] + log2f(lt) : -INFINITY;
            }
          }
        }
        tc_fence_before();
        named_sync(1, 128);
        mbar_arrive(bar(kBarOEmpty + (seg & 1)));
      }
    }
  }

  // ---- teardown --------------------------------------------------------------
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  __syncwarp();
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(Lay::kTmemCols)
                 : "memory");
}

// ---- host side ------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

template <int DT, int P8>
int launch_tc(const TcParams &tp, int smem, cudaStream_t st) {
  auto k = partial_tcgen05_kernel<DT, P8>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return (int)e;
  k<<<tp.n_ctas, kThreads, smem, st>>>(tp);
  return (int)cudaGetLastError();
}

template <int DT>
int launch_tc_p(const TcParams &tp, int p8, int smem, cudaStream_t st) {
  switch (p8) {
    case 8: return launch_tc<DT, 8>(tp, smem, st);
    case 16: return launch_tc<DT, 16>(tp, smem, st);
    case 24: return launch_tc<DT, 24>(tp, smem, st);
    case 32: return launch_tc<DT, 32>(tp, smem, st);
    case 48: return launch_tc<DT, 48>(tp, smem, st);
  }
  return (int)cudaErrorInvalidValue;
}

int smem_for(int p8, int stages) {
  switch (p8) {
    case 8: return TcLayout<8>::smem_bytes(stages);
    case 16: return TcLayout<16>::smem_bytes(stages);
    case 24: return TcLayout<24>::smem_bytes(stages);
    case 32: return TcLayout<32>::smem_bytes(stages);
    case 48: return TcLayout<48>::smem_bytes(stages);
  }
  return -1;
}

}  // namespace

int lse_tc_pairs_bucket(int pairs) {
  if (pairs <= 8) return 8;
  if (pairs <= 16) return 16;
  if (pairs <= 24) return 24;
  if (pairs <= 32) return 32;
  if (pairs <= 48) return 48;
  return -1;
}

int lse_tc_smem(int p8, int smem_optin, int *stages) {
  int best = -1;
  for (int ns = 2; ns <= 4; ++ns) {
    const int b = smem_for(p8, ns);
    if (b > 0 && b <= smem_optin) {
      best = b;
      *stages = ns;
    }
  }
  return best;
}

int lse_tc_key_tile() { return kTK; }

int lse_tc_build_maps(const uint64_t *chunk_base, int n_chunks, size_t chunk_bytes,
                      int n_kv_heads, int box_tokens, void *maps_out) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = get_encode();
  if (!enc) return (int)cudaErrorNotSupported;
  if (n_chunks > LSE_MAX_TMA_CHUNKS) return (int)cudaErrorInvalidValue;
  CUtensorMap *maps = static_cast<CUtensorMap *>(maps_out);
  const uint64_t row = (uint64_t)n_kv_heads * kD * 2;  // bytes per token, all kv heads
  for (int c = 0; c < n_chunks; ++c) {
    cuuint64_t dims[3] = {64, (cuuint64_t)n_kv_heads * 2, (cuuint64_t)(chunk_bytes / row)};
    cuuint64_t strides[2] = {128, row};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)box_tokens};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(&maps[c], CU_TENSOR_MAP_DATA_TYPE_UINT16, 3,
                     reinterpret_cast<void *>(chunk_base[c]), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return (int)cudaErrorInvalidValue;
  }
  return 0;
}

size_t lse_tc_map_bytes() { return sizeof(CUtensorMap); }

int lse_launch_partial_tcgen05(const LseKernelParams &p, const void *maps, int n_maps,
                               int dtype, int p8, int n_ctas, int n_slots, int stages,
                               int box_tokens, int smem, void *stream) {
  static_assert(sizeof(TcParams) < 30000, "kernel parameter block too large");
  TcParams tp;
  memset(&tp, 0, sizeof tp);
  memcpy(tp.maps, maps, sizeof(CUtensorMap) * n_maps);
  tp.p = p;
  tp.n_ctas = n_ctas;
  tp.n_slots = n_slots;
  tp.stages = stages;
  tp.box_tokens = box_tokens;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  switch (dtype) {
    case LSE_KV_BF16: return launch_tc_p<LSE_KV_BF16>(tp, p8, smem, st);
    case LSE_KV_F16: return launch_tc_p<LSE_KV_F16>(tp, p8, smem, st);
  }
  return (int)cudaErrorInvalidValue;
}
