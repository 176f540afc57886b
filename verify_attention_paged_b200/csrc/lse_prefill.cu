// Tensor-core (tcgen05) pass for long query blocks, sm_100a.
//
// What it computes is the paged attention of a block of query rows that is
// longer than a verify step: the LSE releases page (v0.4.14, "Improvements")
// describes a WMMA paged-attention kernel for such blocks (prefill chunks of
// up to 1024 rows) that skips 256-key windows no row of the block sees,
// while the windows that contribute keep their arithmetic.  Here every row
// r of sequence s (position C_s + r, C_s = L_s - R_s) sees the keys 0 ..
// C_s + r (the chain of a block, no tree masks), exactly as the verify
// passes define it.
//
// How it is computed on B200:
//
//  * Rows are the M of both products: a work unit (segment) is one query
//    head of one 128-row tile of one sequence; S = Q K^T (M = 128 rows, N =
//    128 keys) and O = P V (M = 128 rows, N = 128 dims) accumulate in FP32
//    in TMEM.  One softmax thread per row (the row's TMEM lane) holds its
//    running maximum and sum.
//  * A segment's key loop ends at the tile holding the last key its last
//    row sees: 128-key tiles past it are never enumerated, never loaded and
//    never multiplied (the pages skip 256-key windows; the skip here is at
//    the 128-key tile, which skips every such window and more).  Keys inside
//    the last tiles that some rows do not see are masked per element.
//  * Operand precision as in the verify pass: with 16-bit K/V, Q and P carry
//    a hi + lo pair of 16-bit terms (two MMAs per K step, accumulated into the
//    same columns); with FP8 K/V, Q enters as four E4M3 terms under a per-row
//    power-of-2 scale and P (times 2^7) as four E5M2 terms of its F16
//    rounding.  P is written back over the score columns it came from and
//    read by the output product straight from TMEM (A operand in TMEM).
//  * Persistent grid, one CTA per SM: the key tiles of all segments are laid
//    end to end and cut into equal contiguous ranges.  A segment covered by
//    one CTA is written to the output directly; the pieces of a segment that
//    several CTAs share are merged at the end of the launch (log-sum-exp
//    weights) by those CTAs, after a bounded wait for the others' partials
//    (a cooperative launch, so all CTAs are resident).
//  * Roles (320 threads): warp 0 streams K and V tiles through the page
//    table by TMA, warp 1 issues the MMAs (and owns TMEM), and two groups of
//    four warps (2-5 and 6-9) stage each segment's Q, run the softmax and
//    write the results: thread r of each group holds row r, the first group
//    the tile's keys 0-63 (and head dims 0-63 of the output), the second
//    keys 64-127 (dims 64-127); the groups meet at named barriers to share
//    each row's maximum and sum.
//    Every wait is bounded and reports LSE_DEVERR_TIMEOUT when it runs out.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cstdint>
#include <cstring>

#include "lse_internal.h"
#include "lse_smem_attr.h"
#include "lse_tc_ptx.h"

namespace {

using namespace lse_ptx;

constexpr int kTK = 128;        // keys per tile = N of the score product
constexpr int kRT = 128;        // query rows per tile = M of both products
constexpr int kD = 128;         // head dim = N of the output product
constexpr int kThreads = 320;
constexpr float kTau = 8.f;     // lazy-rescale threshold (log2 units)
constexpr int kRegion = 128 * 128;  // 128 rows x 128 bytes
constexpr int kQBytes = 4 * kRegion;  // Q terms: 16-bit hi | lo (two regions each), or 4 FP8
constexpr int kPScaleLog2 = 7;  // FP8: P enters the products times 2^7
constexpr int kRowTab = 256;    // row tiles a launch can hold in its table
constexpr int kMaxStagesPf = 6;

struct __align__(64) PfParams {
  CUtensorMap maps[LSE_MAX_TMA_CHUNKS];
  LseKernelParams p;
  int n_ctas;
  int stages;
  int box_tokens;
  int fused;  // always 1 for this pass: it writes p.out / p.lse_out
};

// One 128-row tile of one sequence, for all query heads.
struct RowTile {
  int prefix;      // global index of the first key tile of its first segment (head 0)
  int n_kt;        // key tiles of each of its segments
  int seg_prefix;  // index of its head-0 segment among all segments
  int seq, L, C;   // the sequence, its keys and context length
  int row0;        // call row of the sequence's row 0
  int r0, rows;    // first row of the tile within the sequence, rows in the tile
};

struct EndRecP {
  int seg_id, n_pieces, piece, rt, h;
  long long seg_first;
};

constexpr bool is_f8(int dt) { return dt == LSE_KV_FP8_E4M3 || dt == LSE_KV_FP8_E5M2; }

// K/V stage: 128 keys x 128 dims of one kv head (two 64-dim regions when
// 16-bit, one 128-dim region when 8-bit).
__host__ __device__ constexpr int half_stage(int dt) { return is_f8(dt) ? kRegion : 2 * kRegion; }

enum {
  kFullK = 0,    // [8]
  kEmptyK = 8,   // [8]
  kFullV = 16,   // [8]
  kEmptyV = 24,  // [8]
  kSFull = 32,   // [2] score buffer complete
  kPFull = 34,   // [2] probabilities written over the score buffer (256 arrivals)
  kPvDone = 36,  // [2] output product of a tile of this parity complete
  kQFull = 38,   // Q of a segment staged (256 arrivals)
  kQEmpty = 39,  // the segment's score products complete (Q may be replaced)
  kOFull = 40,   // the piece's last output product complete
  kOEmpty = 41,  // the piece's output read out (256 arrivals)
  kDoneMma = 42, // every MMA issued has completed
  kInfo = 43,    // [8] tile records
  kBarsPf = 56,
};

// exchange of the two softmax groups: per row, partial maxima [2 tiles][2
// groups][128], partial sums [2 groups][128], Q maxima [2 groups][128]
constexpr int kXchBytes = (2 * 2 * 128 + 2 * 128 + 2 * 128) * 4;
constexpr int kMiscPf = kBarsPf * 8 + 16 + 8 * 16 + 2 * 32 * 16 * 4 + kRowTab * (int)sizeof(RowTile) +
                        2 * (int)sizeof(EndRecP) + 64 + kXchBytes;

int prefill_smem_bytes(int dt, int stages) {
  return 1024 + kQBytes + stages * 2 * half_stage(dt) + kMiscPf;
}

// Key tiles a row tile's segments read: up to the last key its last row sees.
__device__ __forceinline__ int row_tile_keys(int C, int r_end) { return (C + r_end + kTK - 1) / kTK; }

// Walks a CTA's contiguous range of global key tiles: row tile (table
// entry), query head, key tile.
struct PfIter {
  int rt, h, kt, n_kt, seg_id;
  long long seg_first, t, t_end;
  const RowTile *tab;
  int n_rt, Hq;
  __device__ void init(const RowTile *table, int n_rows_tiles, int n_heads, long long t0,
                       long long t1) {
    tab = table;
    n_rt = n_rows_tiles;
    Hq = n_heads;
    t = t0;
    t_end = t1;
    rt = h = kt = n_kt = seg_id = 0;
    seg_first = 0;
    if (t >= t_end) return;
    int lo = 0, hi = n_rt - 1;  // last row tile whose first tile is at or before t
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if ((long long)tab[mid].prefix <= t) lo = mid;
      else hi = mid - 1;
    }
    // skip row tiles without keys (none exist: every tile has a key)
    rt = lo;
    n_kt = tab[rt].n_kt;
    const long long off = t - tab[rt].prefix;
    h = int(off / n_kt);
    kt = int(off - (long long)h * n_kt);
    seg_first = tab[rt].prefix + (long long)h * n_kt;
    seg_id = tab[rt].seg_prefix + h;
  }
  __device__ bool valid() const { return t < t_end; }
  __device__ bool seg_start(long long t_begin) const { return t == t_begin || kt == 0; }
  __device__ bool seg_end() const { return t == t_end - 1 || kt == n_kt - 1; }
  __device__ void advance() {
    ++t;
    if (t >= t_end) return;
    if (++kt == n_kt) {
      kt = 0;
      seg_first += n_kt;
      ++seg_id;
      if (++h == Hq) {
        h = 0;
        ++rt;
        n_kt = tab[rt].n_kt;
      }
    }
  }
};

__device__ __forceinline__ int cta_of(long long t, long long U, int C) {
  return int(((t + 1) * (long long)C - 1) / U);
}

// Fragment ids of the boxes of key tile kt of a sequence (-1 past L, -2 a
// bad entry, flagged).
__device__ __noinline__ void pf_page_ids(const LseKernelParams &p, int seq, int kt, int L, int nbox,
                                         int box_t, int *pk, int *pv) {
  const int key0 = kt * kTK;
  const int T = p.tokens_per_fragment;
#pragma unroll 1
  for (int b = 0; b < nbox; ++b) {
    const int kb = key0 + b * box_t;
    int fk = -1, fv = -1;
    if (kb < L) {
      const long long e = (long long)seq * p.max_pages + kb / T;
      fk = p.k_pages[e];
      fv = p.v_pages[e];
      const bool bk = fk < 0 || fk >= p.n_fragments, bv = fv < 0 || fv >= p.n_fragments;
      if (bk || bv) atomicOr(p.err, LSE_DEVERR_BAD_FRAGMENT);
      if (bk) fk = -2;
      if (bv) fv = -2;
    }
    pk[b] = fk;
    pv[b] = fv;
  }
}

__device__ __forceinline__ void pf_boxes(const PfParams &tp, int nbox, int box_t, int regions,
                                         int g, int key0, const int *ids, uint32_t dst,
                                         uint32_t bar) {
  const LseKernelParams &p = tp.p;
  const int T = p.tokens_per_fragment;
#pragma unroll 1
  for (int b = 0; b < nbox; ++b) {
    const int f = ids[b];
    if (f < 0) continue;
    const int kb = key0 + b * box_t;
    const int c = f / p.frags_per_chunk;
    const int z = (f - c * p.frags_per_chunk) * T + kb % T;
#pragma unroll 1
    for (int r = 0; r < regions; ++r)
      tma_load_3d(dst + b * box_t * 128 + r * kRegion, &tp.maps[c], bar, 0, g * regions + r, z);
  }
}

// tcgen05.mma with the A operand in TMEM (the probabilities).
__device__ __forceinline__ void mma_f16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                           uint32_t idesc, uint32_t accumulate, uint32_t leader) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.ne.b32 e, %5, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate), "r"(leader)
      : "memory");
}
__device__ __forceinline__ void mma_f8_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                          uint32_t idesc, uint32_t accumulate, uint32_t leader) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.ne.b32 e, %5, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate), "r"(leader)
      : "memory");
}

// TMEM stores of 32 consecutive columns of this thread's lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t *v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

// Stage dims 64 kh .. 64 kh + 63 of row r of a segment's Q (FP32 times the
// softmax scale in log2 units) into the score product's operand layout:
// 16-bit, hi and lo terms of the 64-dim region kh; FP8, four E4M3 terms under
// the row's power-of-2 scale 2^e (max |x| 2^e in [128, 256) over all 128
// dims: the two groups' maxima meet in qmax), whose inverse is returned.
// Rows past the sequence's rows are zero.
template <int DT>
__device__ __forceinline__ float pf_stage_q(const LseKernelParams &p, const float *src, bool live,
                                            int r, int kh, uint8_t *qs, float *qmax, int bar_id) {
  const float sc = p.scale_log2;
  float isig = 1.f;
  if constexpr (is_f8(DT)) {
    float mx = 0.f;
    if (live) {
#pragma unroll 4
      for (int c = 0; c < 16; ++c) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(src) + 16 * kh + c);
        mx = fmaxf(mx, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
      }
    }
    qmax[kh * 128 + r] = mx;
    named_sync(bar_id, 256);
    mx = fmaxf(qmax[r], qmax[128 + r]) * fabsf(sc);
    int e = 0;
    if (mx > 0.f && mx <= FLT_MAX) {
      const int E = ((__float_as_int(mx) >> 23) & 0xff) - 127;
      e = min(max(7 - E, -126), 126);
    }
    const float sg = sc * exp2i(e);
    isig = exp2i(-e);
#pragma unroll 1
    for (int c = 8 * kh; c < 8 * kh + 8; ++c) {  // 8-dim chunk c = dims 8c .. 8c + 7
      float x[8];
      if (live) {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(src) + 2 * c);
        const float4 b = __ldg(reinterpret_cast<const float4 *>(src) + 2 * c + 1);
        x[0] = a.x * sg; x[1] = a.y * sg; x[2] = a.z * sg; x[3] = a.w * sg;
        x[4] = b.x * sg; x[5] = b.y * sg; x[6] = b.z * sg; x[7] = b.w * sg;
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = 0.f;
      }
      uint2 w[4];
      f8_terms<false, 4>(x, w);
      const uint32_t off = r * 128 + (((c >> 1) ^ (r & 7)) << 4) + (c & 1) * 8;
#pragma unroll
      for (int t = 0; t < 4; ++t) *reinterpret_cast<uint2 *>(qs + t * kRegion + off) = w[t];
    }
  } else {
#pragma unroll 1
    for (int c = 8 * kh; c < 8 * kh + 8; ++c) {
      uint4 vh = make_uint4(0, 0, 0, 0), vl = make_uint4(0, 0, 0, 0);
      if (live) {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(src) + 2 * c);
        const float4 b = __ldg(reinterpret_cast<const float4 *>(src) + 2 * c + 1);
        split2<DT>(a.x * sc, a.y * sc, vh.x, vl.x);
        split2<DT>(a.z * sc, a.w * sc, vh.y, vl.y);
        split2<DT>(b.x * sc, b.y * sc, vh.z, vl.z);
        split2<DT>(b.z * sc, b.w * sc, vh.w, vl.w);
      }
      const int region = c >> 3, cc = c & 7;
      const uint32_t off = region * kRegion + r * 128 + ((cc ^ (r & 7)) << 4);
      *reinterpret_cast<uint4 *>(qs + off) = vh;
      *reinterpret_cast<uint4 *>(qs + 2 * kRegion + off) = vl;
    }
  }
  return isig;
}

// End phase: this CTA's share of each segment it shares with other CTAs
// (the partials of CTA c sit in slot 0 when the segment is c's first, else
// slot 1).
__device__ __noinline__ void pf_end_merge(const PfParams &tp, const RowTile *tab, const EndRecP *rec,
                                          int n_rec, long long U, int C, volatile int *abort_flag,
                                          int *go_flag) {
  const LseKernelParams &p = tp.p;
  const int tid = threadIdx.x;
  const long long slot_stride = (long long)kRT * kD;
#pragma unroll 1
  for (int k = 0; k < n_rec; ++k) {
    const EndRecP r = rec[k];
    unsigned int *cnt = p.seg_count + 2 * r.seg_id;
    if (tid == 0) {
      int go = *abort_flag == 0;
      const long long t0 = clock64();
      while (go) {
        unsigned int v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(cnt) : "memory");
        if (v >= (unsigned)r.n_pieces) break;
        if (clock64() - t0 > kWaitCycles) {
          *abort_flag = 1;
          atomicOr(p.err, LSE_DEVERR_TIMEOUT);
          go = 0;
        }
        __nanosleep(256);
      }
      *go_flag = go;
    }
    __syncthreads();
    const bool go = *go_flag != 0;
    if (go) {
      const RowTile &rt = tab[r.rt];
      const int c_first = cta_of(r.seg_first, U, C);
      const long long E = (long long)rt.rows * kD;
      const long long e0 = E * r.piece / r.n_pieces, e1 = E * (r.piece + 1) / r.n_pieces;
#pragma unroll 1
      for (long long e = e0 + tid; e < e1; e += kThreads) {
        const int row = (int)(e / kD), d = (int)(e - (long long)row * kD);
        float M = -INFINITY;
#pragma unroll 1
        for (int i = 0; i < r.n_pieces; ++i) {
          const int c = c_first + i;
          const int slot = U * c / C >= r.seg_first ? 0 : 1;
          M = fmaxf(M, __ldcg(p.lse_part + ((long long)c * 2 + slot) * kRT + row));
        }
        float W = 0.f, acc = 0.f;
        if (M != -INFINITY) {
#pragma unroll 1
          for (int i = 0; i < r.n_pieces; ++i) {
            const int c = c_first + i;
            const int slot = U * c / C >= r.seg_first ? 0 : 1;
            const long long pi = (long long)c * 2 + slot;
            const float l = __ldcg(p.lse_part + pi * kRT + row);
            const float w = l == -INFINITY ? 0.f : ex2(l - M);
            W += w;
            acc = fmaf(w, __ldcg(p.o_part + pi * slot_stride + (long long)row * kD + d), acc);
          }
        }
        const long long oi = (long long)(rt.row0 + rt.r0 + row) * p.n_q_heads + r.h;
        p.out[oi * kD + d] = W > 0.f ? acc * rcp(W) : 0.f;
        if (d == 0 && p.lse_out)
          p.lse_out[oi] = W > 0.f ? (M + lg2(W)) * 0.69314718055994530942f : -INFINITY;
      }
    }
    __syncthreads();
    if (tid == 0 && go) {
      const unsigned int left = atomicAdd(cnt + 1, 1u);
      if (left + 1u == (unsigned)r.n_pieces) {
        atomicExch(cnt, 0u);
        atomicExch(cnt + 1, 0u);
      }
    }
  }
}

template <int DT>
__global__ void __launch_bounds__(kThreads, 1) prefill_tcgen05_kernel(const __grid_constant__ PfParams tp) {
  constexpr bool kF8 = is_f8(DT);
  constexpr bool kE5 = DT == LSE_KV_FP8_E5M2;
  constexpr int kHalf = half_stage(DT);
  const LseKernelParams &p = tp.p;
  const int NS = tp.stages;
  const int cta = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t q_base = sbase;                    // Q terms (64 KB)
  const uint32_t k_base = q_base + kQBytes;         // K ring
  const uint32_t v_base = k_base + NS * kHalf;      // V ring
  uint8_t *misc = smem + kQBytes + 2 * NS * kHalf;
  uint64_t *bars = reinterpret_cast<uint64_t *>(misc);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + kBarsPf * 8);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + kBarsPf * 8 + 4);
  long long *shared_u = reinterpret_cast<long long *>(misc + kBarsPf * 8 + 8);
  uint4 *tile_info = reinterpret_cast<uint4 *>(misc + kBarsPf * 8 + 16);       // [8]
  int *page_buf = reinterpret_cast<int *>(tile_info + 8);                       // [2][32][16]
  RowTile *tab = reinterpret_cast<RowTile *>(page_buf + 2 * 32 * 16);           // [kRowTab]
  EndRecP *end_rec = reinterpret_cast<EndRecP *>(tab + kRowTab);                // [2]
  int *n_end = reinterpret_cast<int *>(end_rec + 2);
  int *go_flag = n_end + 1;
  int *n_rt_sh = n_end + 2;
  float *xch_m = reinterpret_cast<float *>(n_end + 16);  // [2 tiles][2 groups][128]
  float *xch_l = xch_m + 2 * 2 * 128;                   // [2 groups][128]
  float *xch_q = xch_l + 2 * 128;                       // [2 groups][128]
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // ---- prologue: the row-tile table (warp 0), barriers ----
  if (warp == 0) {
    // lane l takes sequences [l per, (l+1) per); a warp scan of row tiles and
    // key tiles gives each row tile its first key tile
    const int per = (p.n_seqs + 31) / 32;
    const int s0 = min(p.n_seqs, lane * per), s1 = min(p.n_seqs, s0 + per);
    int my_rt = 0;
    long long my_tiles = 0;
    bool bad = false;
    for (int s = s0; s < s1; ++s) {
      const int L = p.seq_lens[s], row0 = p.row_offsets[s], R = p.row_offsets[s + 1] - row0;
      const long long cap = (long long)p.max_pages * p.tokens_per_fragment;
      if (row0 < 0 || R < 0 || R > p.max_rows || row0 + R > p.max_total_rows || R > L ||
          (long long)L > cap) {
        bad = true;
        continue;
      }
      const int nrt = (R + kRT - 1) / kRT;
      my_rt += nrt;
      for (int t = 0; t < nrt; ++t)
        my_tiles += (long long)row_tile_keys(L - R, min(R, (t + 1) * kRT)) * p.n_q_heads;
    }
    int rt_incl = my_rt;
    long long tiles_incl = my_tiles;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, rt_incl, o);
      const long long b = __shfl_up_sync(0xffffffffu, tiles_incl, o);
      if (lane >= o) {
        rt_incl += a;
        tiles_incl += b;
      }
    }
    int idx = rt_incl - my_rt;
    long long run = tiles_incl - my_tiles;
    for (int s = s0; s < s1; ++s) {
      const int L = p.seq_lens[s], row0 = p.row_offsets[s], R = p.row_offsets[s + 1] - row0;
      const long long cap = (long long)p.max_pages * p.tokens_per_fragment;
      if (row0 < 0 || R < 0 || R > p.max_rows || row0 + R > p.max_total_rows || R > L ||
          (long long)L > cap)
        continue;
      const int nrt = (R + kRT - 1) / kRT;
      for (int t = 0; t < nrt; ++t, ++idx) {
        const int r_end = min(R, (t + 1) * kRT);
        const int n_kt = row_tile_keys(L - R, r_end);
        if (idx < kRowTab)
          tab[idx] = RowTile{(int)run, n_kt, idx * p.n_q_heads, s, L, L - R, row0, t * kRT,
                             r_end - t * kRT};
        run += (long long)n_kt * p.n_q_heads;
      }
    }
    bad = __any_sync(0xffffffffu, bad);
    const int total_rt = __shfl_sync(0xffffffffu, rt_incl, 31);
    if (lane == 31) *shared_u = tiles_incl;
    if (lane == 0) {
      *n_rt_sh = total_rt;
      if (cta == 0 && bad) atomicOr(p.err, LSE_DEVERR_BAD_LENGTH);
      // (the planner keeps row tiles within the table; a call past it is refused here)
      if (cta == 0 && total_rt > kRowTab) atomicOr(p.err, LSE_DEVERR_BAD_LENGTH);
    }
  }
  if (tid == 32) {
    *abort_flag = 0;
    for (int i = 0; i < 8; ++i) {
      mbar_init(bar(kFullK + i), 1);
      mbar_init(bar(kEmptyK + i), 1);
      mbar_init(bar(kFullV + i), 1);
      mbar_init(bar(kEmptyV + i), 1);
      mbar_init(bar(kInfo + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kSFull + i), 1);
      mbar_init(bar(kPFull + i), 256);
      mbar_init(bar(kPvDone + i), 1);
    }
    mbar_init(bar(kQFull), 256);
    mbar_init(bar(kQEmpty), 1);
    mbar_init(bar(kOFull), 1);
    mbar_init(bar(kOEmpty), 256);
    mbar_init(bar(kDoneMma), 1);
    *n_end = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const long long U = *shared_u;
  const int n_rt = *n_rt_sh;
  const int C = (int)(U < tp.n_ctas ? U : tp.n_ctas);
  if (cta >= C || n_rt > kRowTab) {
    if (warp == 1)
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512)
                   : "memory");
    return;
  }
  const long long t_begin = U * cta / C, t_stop = U * (cta + 1) / C;
  const int n_total = (int)(t_stop - t_begin);
  const int box_t = tp.box_tokens;
  const int nbox = box_t >= kTK ? 1 : kTK / box_t;
  const uint32_t full_boxes = nbox >= 32 ? 0xffffffffu : ((1u << nbox) - 1u);
  const int G = p.group;
  const int Hq = p.n_q_heads;
  // TMEM: score / probability buffers at columns 0 and 128, output at 256
  auto tmem_s = [&](int buf) { return tmem + (uint32_t)(buf * 128); };
  const uint32_t tmem_o = tmem + 256u;

  if (warp == 0) {
    // ============================ TMA producer ============================
    int *pk = page_buf, *pv = page_buf + 32 * 16;
    int n = 0;
    bool ok = true;
#pragma unroll 1
    for (int b0 = 0; b0 < n_total && ok; b0 += 32) {
      const int cnt = n_total - b0 < 32 ? n_total - b0 : 32;
      PfIter mine;
      mine.init(tab, n_rt, Hq, t_begin + b0 + (lane < cnt ? lane : 0), t_stop);
      if (lane < cnt) {
        const RowTile &rt = tab[mine.rt];
        pf_page_ids(p, rt.seq, mine.kt, rt.L, nbox, box_t, pk + lane * 16, pv + lane * 16);
      }
      __syncwarp();
#pragma unroll 1
      for (int i = 0; i < cnt; ++i, ++n) {
        const int t_rt = __shfl_sync(0xffffffffu, mine.rt, i);
        const int t_h = __shfl_sync(0xffffffffu, mine.h, i);
        const int t_kt = __shfl_sync(0xffffffffu, mine.kt, i);
        int go = 1;
        if (lane == 0) {
          const int st = n % NS;
          const uint32_t ph = ((n / NS) & 1) ^ 1;
          const int L = tab[t_rt].L;
          const int key0 = t_kt * kTK;
          const int *ik = pk + i * 16, *iv = pv + i * 16;
          uint32_t kmask = 0, vmask = 0;
          for (int b = 0; b < nbox; ++b) {
            if (ik[b] >= 0) kmask |= 1u << b;
            if (iv[b] >= 0) vmask |= 1u << b;
          }
          const int live = L - key0 < kTK ? L - key0 : kTK;
          const uint32_t box_bytes = (uint32_t)(kF8 ? 1 : 2) * (uint32_t)box_t * 128u;
          const int g = t_h / G;
          go = mbar_wait(bar(kEmptyK + st), ph, abort_flag, p.err);
          if (go) {
            tile_info[n & 7] = make_uint4(kmask, vmask, (uint32_t)live, 0u);
            mbar_arrive(bar(kInfo + (n & 7)));
            mbar_expect_tx(bar(kFullK + st), (uint32_t)__popc(kmask) * box_bytes);
            pf_boxes(tp, nbox, box_t, kF8 ? 1 : 2, g, key0, ik, k_base + st * kHalf,
                     bar(kFullK + st));
            go = mbar_wait(bar(kEmptyV + st), ph, abort_flag, p.err);
          }
          if (go) {
            mbar_expect_tx(bar(kFullV + st), (uint32_t)__popc(vmask) * box_bytes);
            pf_boxes(tp, nbox, box_t, kF8 ? 1 : 2, g, key0, iv, v_base + st * kHalf,
                     bar(kFullV + st));
          }
        }
        go = __shfl_sync(0xffffffffu, go, 0);
        if (!go) {
          ok = false;
          break;
        }
      }
      __syncwarp();
    }
    if (lane == 0)
#pragma unroll 1
      for (int k = (n > NS ? n - NS : 0); k < n; ++k) {
        mbar_drain(bar(kFullK + k % NS), (k / NS) & 1);
        mbar_drain(bar(kFullV + k % NS), (k / NS) & 1);
      }
  } else if (warp == 1) {
    // ============================ MMA issuer ============================
    // Order per tile n: S(n), then P(n-1) V; at a segment start the previous
    // segment's last output product goes first (its epilogue must not wait
    // on this segment's Q).  S(n) reuses the buffer of P(n-2), so it waits
    // for that output product to complete.
    constexpr uint32_t f16fmt = DT == LSE_KV_BF16 ? 1u : 0u;
    constexpr uint32_t kvfmt = kF8 ? (kE5 ? 1u : 0u) : f16fmt;
    constexpr uint32_t idesc_s = instr_desc(kF8 ? 0u : f16fmt, kvfmt, 0, 0, kRT, kTK);
    constexpr uint32_t idesc_o = instr_desc(kF8 ? 1u : f16fmt, kvfmt, 0, 1, kRT, kD);
    const uint32_t leader = elect_one();
    PfIter it;
    it.init(tab, n_rt, Hq, t_begin, t_stop);
    int seg = -1, pv_seg = -1;
    bool ok = true;
    bool pv_first = true;  // the next output product starts its piece's accumulator
    auto issue_pv = [&](int m, bool last_of_piece) -> bool {
      // P(m) V(m) into O
      bool go = mbar_wait(bar(kPFull + (m & 1)), (m >> 1) & 1, abort_flag, p.err);
      go = go && mbar_wait(bar(kFullV + m % NS), (m / NS) & 1, abort_flag, p.err);
      if (go && pv_first && pv_seg > 0)
        go = mbar_wait(bar(kOEmpty), (pv_seg - 1) & 1, abort_flag, p.err);
      if (!__all_sync(0xffffffffu, go)) return false;
      tc_fence_after();
      const uint32_t vaddr = v_base + (m % NS) * kHalf;
      const uint32_t pa = tmem_s(m & 1);
      if constexpr (kF8) {
        const uint64_t b0 = smem_desc(vaddr, 0, 1024, kLayoutSw128);
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
          for (int k = 0; k < kTK / 32; ++k)
            mma_f8_ta(tmem_o, pa + (uint32_t)(32 * t + 8 * k), b0 + (uint64_t)(k * 4096 / 16),
                      idesc_o, (pv_first && t == 0 && k == 0) ? 0u : 1u, leader);
      } else {
        const uint64_t b0 = smem_desc(vaddr, kRegion, 1024, kLayoutSw128);
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int k = 0; k < kTK / 16; ++k)
            mma_f16_ta(tmem_o, pa + (uint32_t)(64 * t + 8 * k), b0 + (uint64_t)(k * 2048 / 16),
                       idesc_o, (pv_first && t == 0 && k == 0) ? 0u : 1u, leader);
      }
      mma_commit(bar(kEmptyV + m % NS), leader);
      mma_commit(bar(kPvDone + (m & 1)), leader);
      pv_first = false;
      if (last_of_piece) {
        mma_commit(bar(kOFull), leader);
        pv_first = true;
      }
      return true;
    };
    bool prev_last = false;  // tile n - 1 ended its piece
#pragma unroll 1
    for (int n = 0; n < n_total; ++n, it.advance()) {
      const bool first = it.seg_start(t_begin), last = it.seg_end();
      if (first) ++seg;
      if (first && n > 0) {
        if (!issue_pv(n - 1, prev_last)) { ok = false; break; }
      }
      if (first) pv_seg = seg;
      // S(n): the segment's Q, K(n), and the buffer's previous P consumed
      bool go = !first || mbar_wait(bar(kQFull), seg & 1, abort_flag, p.err);
      go = go && mbar_wait(bar(kFullK + n % NS), (n / NS) & 1, abort_flag, p.err);
      go = go && (n < 2 || mbar_wait(bar(kPvDone + (n & 1)), ((n - 2) >> 1) & 1, abort_flag, p.err));
      if (!__all_sync(0xffffffffu, go)) { ok = false; break; }
      tc_fence_after();
      const uint32_t kaddr = k_base + (n % NS) * kHalf;
      const uint32_t d = tmem_s(n & 1);
      if constexpr (kF8) {
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_f8(d, smem_desc(q_base + t * kRegion + k * 32, 16, 1024, kLayoutSw128),
                   smem_desc(kaddr + k * 32, 16, 1024, kLayoutSw128), idesc_s,
                   (t | k) ? 1u : 0u, leader);
      } else {
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t off = (k >> 2) * kRegion + (k & 3) * 32;
            mma_f16(d, smem_desc(q_base + t * 2 * kRegion + off, 16, 1024, kLayoutSw128),
                    smem_desc(kaddr + off, 16, 1024, kLayoutSw128), idesc_s, (t | k) ? 1u : 0u,
                    leader);
          }
      }
      mma_commit(bar(kEmptyK + n % NS), leader);
      mma_commit(bar(kSFull + (n & 1)), leader);
      if (last) mma_commit(bar(kQEmpty), leader);
      if (!first && n > 0) {
        if (!issue_pv(n - 1, prev_last)) { ok = false; break; }
      }
      prev_last = last;
    }
    if (ok && n_total > 0) issue_pv(n_total - 1, true);
    mma_commit(bar(kDoneMma), leader);
    mbar_drain(bar(kDoneMma), 0);
  } else {
    // ====== Q staging, softmax and epilogue: warps 2-5 (keys 0-63) and 6-9 (64-127) ======
    const int kh = (warp - 2) >> 2;               // key half of the tile, head-dim half of O
    const int quarter = warp & 3;                 // TMEM lane quarter
    const int r = quarter * 32 + lane;            // the row of the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    constexpr int kBar = 1;                       // named barrier of these 256 threads
    constexpr int kHK = kTK / 2;                  // keys of a half
    PfIter it;
    it.init(tab, n_rt, Hq, t_begin, t_stop);
    int seg = -1;
    float m_run = -FLT_MAX, l_run = 0.f, isig = 1.f;  // l_run: this half's keys only
    bool had = false, ok = true;
#pragma unroll 1
    for (int n = 0; it.valid() && ok; it.advance(), ++n) {
      const RowTile &rt = tab[it.rt];
      const bool first = it.seg_start(t_begin), last = it.seg_end();
      const bool row_live = r < rt.rows;
      const int pos = rt.C + rt.r0 + r;           // this row's position = last key it sees
      if (first) {
        ++seg;
        // the previous segment's score products are done: replace Q
        bool w = seg == 0 || mbar_wait(bar(kQEmpty), (seg - 1) & 1, abort_flag, p.err);
        if (named_or(kBar, 256, !w)) { ok = false; break; }
        const float *src = p.q + ((long long)(rt.row0 + rt.r0 + r) * Hq + it.h) * kD;
        isig = pf_stage_q<DT>(p, src, row_live, r, kh, smem, xch_q, kBar);
        fence_proxy_async();
        mbar_arrive(bar(kQFull));
        m_run = -FLT_MAX;
        l_run = 0.f;
        had = false;
      }
      // ---- tile n: scores -> probabilities ----
      bool w = mbar_wait(bar(kSFull + (n & 1)), (n >> 1) & 1, abort_flag, p.err);
      w = w && mbar_wait(bar(kInfo + (n & 7)), (n >> 3) & 1, abort_flag, p.err);
      if (named_or(kBar, 256, !w)) { ok = false; break; }
      tc_fence_after();
      const uint4 inf = tile_info[n & 7];
      const int key0 = it.kt * kTK;
      const uint32_t both = inf.x & inf.y;
      const bool tile_full = inf.z == (uint32_t)kTK && both == full_boxes;
      const int kc = kh * kHK;                    // this half's first key in the tile
      float sv[kHK];
#pragma unroll
      for (int c = 0; c < kHK; c += 32) tmem_load<32>(tmem_s(n & 1) + lane_off + kc + c, sv + c);
      if constexpr (kF8) {
#pragma unroll
        for (int j = 0; j < kHK; ++j) sv[j] *= isig;
      }
      // every row of the tile sees every key of this tile?
      const bool all_vis = tile_full && key0 + kTK - 1 <= rt.C + rt.r0;
      if (!all_vis || !row_live) {
#pragma unroll
        for (int j = 0; j < kHK; ++j) {
          const int jj = kc + j;
          const bool vis = row_live && key0 + jj <= pos && jj < (int)inf.z &&
                           ((both >> (jj / box_t)) & 1u);
          if (!vis) sv[j] = -INFINITY;
        }
      }
      float mh = -INFINITY;
#pragma unroll
      for (int j = 0; j < kHK; ++j) mh = fmaxf(mh, sv[j]);
      // the row's maximum over both halves (double-buffered by tile parity)
      float *xm = xch_m + (n & 1) * 256;
      xm[kh * 128 + r] = mh;
      named_sync(kBar, 256);
      const float mx = fmaxf(xm[r], xm[128 + r]);
      const bool need = mx > m_run + kTau;        // the same in both groups
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = need ? mx : m_run;
        const float alpha = ex2(m_run - m_new);
        if (had) {
          // rescale this row's half of the output once the previous output
          // product of the piece has completed (products complete in order)
          const int pn = n - 1;
          const bool wo = mbar_wait(bar(kPvDone + (pn & 1)), (pn >> 1) & 1, abort_flag, p.err);
          if (!__all_sync(0xffffffffu, wo)) { ok = false; }
          if (ok) {
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < kD / 2; c += 8) {
              float v[8];
              tmem_load<8>(tmem_o + lane_off + kh * (kD / 2) + c, v);
#pragma unroll
              for (int i = 0; i < 8; ++i) v[i] *= alpha;
              tmem_st8(tmem_o + lane_off + kh * (kD / 2) + c, v);
            }
            tmem_st_wait();
          }
        }
        l_run *= alpha;
        m_run = m_new;
      }
      if (named_or(kBar, 256, !ok)) { ok = false; break; }
      // probabilities over this half's score columns (A operand of the
      // output product)
      float lsum = 0.f;
      if constexpr (kF8) {
        // P 2^7 as four E5M2 terms of its F16 rounding: term t of keys
        // 4c .. 4c + 3 in column 32 t + c
#pragma unroll
        for (int c0 = 0; c0 < kHK; c0 += 32) {
          uint32_t words[4][8];
#pragma unroll
          for (int c = 0; c < 32; c += 8) {
            float e[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              e[i] = ex2(sv[c0 + c + i] - m_run) * (float)(1 << kPScaleLog2);
              lsum += e[i];
            }
            uint2 wt[4];
            e5_terms_f16<4>(e, wt);
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              words[t][c / 4] = wt[t].x;
              words[t][c / 4 + 1] = wt[t].y;
            }
          }
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            // 8 columns of term t: keys kc + c0 .. kc + c0 + 31
            asm volatile(
                "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(
                    tmem_s(n & 1) + lane_off + (uint32_t)(32 * t + (kc + c0) / 4)),
                "r"(words[t][0]), "r"(words[t][1]), "r"(words[t][2]), "r"(words[t][3]),
                "r"(words[t][4]), "r"(words[t][5]), "r"(words[t][6]), "r"(words[t][7])
                : "memory");
          }
        }
      } else {
        // hi terms in columns 0 .. 63, lo terms in 64 .. 127 (two keys a
        // column): this half's 32 columns of each
        uint32_t hi[32], lo[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float e0 = ex2(sv[2 * c] - m_run), e1 = ex2(sv[2 * c + 1] - m_run);
          lsum += e0 + e1;
          split2<DT>(e0, e1, hi[c], lo[c]);
        }
        tmem_st32(tmem_s(n & 1) + lane_off + (uint32_t)(kc / 2), hi);
        tmem_st32(tmem_s(n & 1) + lane_off + (uint32_t)(64 + kc / 2), lo);
      }
      tmem_st_wait();
      l_run += lsum;
      had = true;
      if (!tile_full) {
        // a V row that holds no live key may hold any bits: zero it (its
        // probability is 0, and 0 x NaN would not be); the first group's
        // thread r takes V row r
        bool wv = true;
        if (kh == 0) {
          wv = mbar_wait(bar(kFullV + n % NS), (n / NS) & 1, abort_flag, p.err);
          const bool dead = !(r < (int)inf.z && ((both >> (r / box_t)) & 1u));
          if (wv && dead) {
            uint8_t *v0 = smem + kQBytes + NS * kHalf + (n % NS) * kHalf + r * 128;
#pragma unroll 1
            for (int c = 0; c < (kF8 ? 8 : 16); ++c)
              *reinterpret_cast<uint4 *>(v0 + (c >> 3) * kRegion + (c & 7) * 16) =
                  make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async();
        }
        if (named_or(kBar, 256, !wv)) { ok = false; break; }
      }
      tc_fence_before();
      mbar_arrive(bar(kPFull + (n & 1)));

      if (last) {
        // ---- epilogue of the piece: this group writes head dims 64 kh .. ----
        bool we = mbar_wait(bar(kOFull), seg & 1, abort_flag, p.err);
        xch_l[kh * 128 + r] = l_run;
        if (named_or(kBar, 256, !we)) { ok = false; break; }
        tc_fence_after();
        const float lt = xch_l[r] + xch_l[128 + r];
        const int c_first = cta_of(it.seg_first, U, C);
        const int c_last = cta_of(it.seg_first + it.n_kt - 1, U, C);
        const int n_pieces = c_last - c_first + 1, piece = cta - c_first;
        const float inv = lt > 0.f ? rcp(lt) : 0.f;
        const float lse2 =
            lt > 0.f ? m_run + lg2(lt) - (kF8 ? (float)kPScaleLog2 : 0.f) : -INFINITY;
        float *dst;
        if (n_pieces == 1) {
          dst = p.out + ((long long)(rt.row0 + rt.r0 + r) * Hq + it.h) * kD;
          if (kh == 0 && row_live && p.lse_out)
            p.lse_out[(long long)(rt.row0 + rt.r0 + r) * Hq + it.h] = lse2 * 0.69314718055994530942f;
        } else {
          const int slot = t_begin >= it.seg_first ? 0 : 1;
          const long long pi = (long long)cta * 2 + slot;
          dst = p.o_part + pi * kRT * kD + (long long)r * kD;
          if (kh == 0) p.lse_part[pi * kRT + r] = row_live ? lse2 : -INFINITY;
        }
#pragma unroll 1
        for (int c = kh * (kD / 2); c < (kh + 1) * (kD / 2); c += 8) {
          float v[8];
          tmem_load<8>(tmem_o + lane_off + c, v);
          if (row_live || n_pieces > 1) {
            float4 a = make_float4(v[0] * inv, v[1] * inv, v[2] * inv, v[3] * inv);
            float4 b = make_float4(v[4] * inv, v[5] * inv, v[6] * inv, v[7] * inv);
            if (!row_live) a = b = make_float4(0.f, 0.f, 0.f, 0.f);
            *reinterpret_cast<float4 *>(dst + c) = a;
            *reinterpret_cast<float4 *>(dst + c + 4) = b;
          }
        }
        tc_fence_before();
        mbar_arrive(bar(kOEmpty));
        if (n_pieces > 1) {
          __threadfence();
          named_sync(kBar, 256);
          if (kh == 0 && r == 0) {
            atomicAdd(p.seg_count + 2 * it.seg_id, 1u);
            const int k = *n_end;
            if (k < 2) {
              end_rec[k] = EndRecP{it.seg_id, n_pieces, piece, it.rt, it.h, it.seg_first};
              *n_end = k + 1;
            }
          }
        }
      }
    }
  }

  // ---- teardown ----
  tc_fence_before();
  __syncthreads();
  pf_end_merge(tp, tab, end_rec, *n_end, U, C, abort_flag, go_flag);
  // TMEM is released last: only its owner fences after the barrier
  if (warp == 1) {
    tc_fence_after();
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512)
                 : "memory");
  }
}

template <int DT>
int launch_pf(const PfParams &tp, int smem, cudaStream_t st) {
  auto k = prefill_tcgen05_kernel<DT>;
  static lse_detail::SmemAllowed allowed;
  const int e = lse_detail::allow_dynamic_smem(k, smem, allowed);
  if (e) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tp.n_ctas);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return (int)cudaLaunchKernelEx(&cfg, k, tp);
}

}  // namespace

int lse_pf_row_tile() { return kRT; }
int lse_pf_max_row_tiles() { return kRowTab; }

// Deepest K/V ring that fits (2 .. 6 stages); -1 when none does.
int lse_pf_smem(int dtype, int smem_optin, int *stages) {
  for (int ns = kMaxStagesPf; ns >= 2; --ns) {
    const int b = prefill_smem_bytes(dtype, ns);
    if (b <= smem_optin) {
      *stages = ns;
      return b;
    }
  }
  return -1;
}

int lse_launch_prefill_tcgen05(const LseKernelParams &p, const void *maps, int n_maps, int dtype,
                               int n_ctas, int stages, int box_tokens, int smem, void *stream) {
  static_assert(sizeof(PfParams) < 30000, "kernel parameter block too large");
  PfParams tp;
  memset(&tp, 0, sizeof tp);
  memcpy(tp.maps, maps, sizeof(CUtensorMap) * n_maps);
  tp.p = p;
  tp.n_ctas = n_ctas;
  tp.stages = stages;
  tp.box_tokens = box_tokens;
  tp.fused = 1;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  switch (dtype) {
    case LSE_KV_BF16: return launch_pf<LSE_KV_BF16>(tp, smem, st);
    case LSE_KV_F16: return launch_pf<LSE_KV_F16>(tp, smem, st);
    case LSE_KV_FP8_E4M3: return launch_pf<LSE_KV_FP8_E4M3>(tp, smem, st);
    case LSE_KV_FP8_E5M2: return launch_pf<LSE_KV_FP8_E5M2>(tp, smem, st);
  }
  return (int)cudaErrorInvalidValue;
}
