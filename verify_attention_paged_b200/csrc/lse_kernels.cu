// CUDA-core partial pass and the log-sum-exp merge pass of split-KV paged
// attention (sm_100a).
//
// Partial pass (LSE releases, v0.4.19 "Long-context split attention": one
// partial family; v0.4.21: K/V reads shared across query heads and rows).
// One CTA per (partition, kv head, sequence).  The CTA streams the
// partition's keys in tiles of 32, reading each K/V row of its kv head once
// through the page table and converting it to FP32 in shared memory; every
// (query row, query head) pair of the group then uses that tile.  Scores,
// online softmax (running max / sum in log2 units) and the P.V accumulation
// run in FP32 on CUDA cores.  A partition past the sequence's live keys
// returns before loading anything (v0.4.20: empty-partition skipping).
//
// Merge pass (v0.4.19: one merge family): for each (row, head) the live
// partials are combined with weights exp(lse_p - max lse).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cfloat>
#include <climits>
#include <cstdint>

#include "lse_internal.h"
#include "lse_smem_attr.h"

namespace {

constexpr int kThreads = 128;
constexpr int kTileKeys = 32;   // keys per tile
constexpr int kPairChunk = 16;  // (row, head) pairs per pass over the keys

// ---- loads and conversions ---------------------------------------------

template <int DT>
struct KvFormat;
template <>
struct KvFormat<LSE_KV_F32> {
  static constexpr int kElemBytes = 4;
  static __device__ __forceinline__ void to_float(const uint4 &v, float *o) {
    o[0] = __uint_as_float(v.x);
    o[1] = __uint_as_float(v.y);
    o[2] = __uint_as_float(v.z);
    o[3] = __uint_as_float(v.w);
  }
};
template <>
struct KvFormat<LSE_KV_F16> {
  static constexpr int kElemBytes = 2;
  static __device__ __forceinline__ void to_float(const uint4 &v, float *o) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __half2 h = *reinterpret_cast<const __half2 *>(&w[i]);
      float2 f = __half22float2(h);
      o[2 * i] = f.x;
      o[2 * i + 1] = f.y;
    }
  }
};
template <>
struct KvFormat<LSE_KV_BF16> {
  static constexpr int kElemBytes = 2;
  static __device__ __forceinline__ void to_float(const uint4 &v, float *o) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162 *>(&w[i]);
      float2 f = __bfloat1622float2(h);
      o[2 * i] = f.x;
      o[2 * i + 1] = f.y;
    }
  }
};
template <__nv_fp8_interpretation_t I>
struct Fp8Format {
  static constexpr int kElemBytes = 1;
  static __device__ __forceinline__ void to_float(const uint4 &v, float *o) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        __nv_fp8x2_storage_t pair = (__nv_fp8x2_storage_t)((w[i] >> (16 * k)) & 0xffffu);
        __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pair, I);
        float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&hr));
        o[4 * i + 2 * k] = f.x;
        o[4 * i + 2 * k + 1] = f.y;
      }
    }
  }
};
template <>
struct KvFormat<LSE_KV_FP8_E4M3> : Fp8Format<__NV_E4M3> {};
template <>
struct KvFormat<LSE_KV_FP8_E5M2> : Fp8Format<__NV_E5M2> {};

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

// Checks shared by both passes; returns false (and flags) on bad lengths.
__device__ __forceinline__ bool seq_shape(const LseKernelParams &p, int s, int &L, int &row0,
                                          int &R) {
  L = p.seq_lens[s];
  row0 = p.row_offsets[s];
  R = p.row_offsets[s + 1] - row0;
  const long long cap = (long long)p.max_pages * p.tokens_per_fragment;
  if (row0 < 0 || R < 0 || R > p.max_rows || row0 + R > p.max_total_rows || R > L ||
      (long long)L > cap) {
    if (threadIdx.x == 0) atomicOr(p.err, LSE_DEVERR_BAD_LENGTH);
    return false;
  }
  return true;
}

// Device address of key `key` of kv head g through a page table, or null
// when the entry names no fragment (flagged).
__device__ __forceinline__ const uint8_t *kv_addr(const LseKernelParams &p, const int32_t *table,
                                                  int s, int key, int g, int row_bytes_head) {
  const int T = p.tokens_per_fragment;
  const int page = key / T;
  const int off = key - page * T;
  const int frag = table[(long long)s * p.max_pages + page];
  if (frag < 0 || frag >= p.n_fragments) {
    atomicOr(p.err, LSE_DEVERR_BAD_FRAGMENT);
    return nullptr;
  }
  const int chunk = frag / p.frags_per_chunk;
  const long long byte = (long long)(frag - chunk * p.frags_per_chunk) * p.fragment_bytes +
                         ((long long)off * p.n_kv_heads + g) * row_bytes_head;
  return reinterpret_cast<const uint8_t *>(p.chunk_base[chunk]) + byte;
}

// Per-vector scale of key `key`, kv head g: entry (g, key % T) of the
// [kv_head][token] scale block of its fragment (the caller has checked the
// page-table entry).
__device__ __forceinline__ float kv_scale(const LseKernelParams &p, const int32_t *table, int s,
                                          int key, int g) {
  const int T = p.tokens_per_fragment;
  const int page = key / T;
  const int frag = table[(long long)s * p.max_pages + page];
  return __ldg(p.scales + ((long long)frag * p.n_kv_heads + g) * T + (key - page * T));
}

// ---- partial pass on CUDA cores ------------------------------------------

template <int D>
struct CcShape {
  static constexpr int kRow = D + 4;  // padded FP32 row in shared memory
  static constexpr int kDimsPerThread = D >= kThreads ? D / kThreads : 1;
  static constexpr int kDimCover = D / kDimsPerThread;     // threads covering D
  static constexpr int kPairSets = kThreads / kDimCover;   // 1 or 2
  static constexpr int kPairsPerThread = kPairChunk / kPairSets;
  static constexpr int kSmemFloats =
      kPairChunk * D + 2 * kTileKeys * kRow + kPairChunk * kTileKeys + 4 * kPairChunk;
  static constexpr int kSmemBytes = kSmemFloats * 4 + kPairChunk * 8;
};

template <int DT, int D>
__global__ void __launch_bounds__(kThreads)
    partial_cuda_core_kernel(const __grid_constant__ LseKernelParams p) {
  using Fmt = KvFormat<DT>;
  using Sh = CcShape<D>;
  constexpr int kEsz = Fmt::kElemBytes;
  constexpr int kVecPerRow = D * kEsz / 16;  // 16-byte vectors per key row
  constexpr int kElemPerVec = 16 / kEsz;

  extern __shared__ __align__(16) unsigned char smem_raw[];
  float *Qs = reinterpret_cast<float *>(smem_raw);  // [PC][D], pre-scaled
  float *Ks = Qs + kPairChunk * D;                   // [TK][kRow]
  float *Vs = Ks + kTileKeys * Sh::kRow;             // [TK][kRow]
  float *Ps = Vs + kTileKeys * Sh::kRow;             // [PC][TK]
  float *alpha_s = Ps + kPairChunk * kTileKeys;      // [PC]
  float *m_s = alpha_s + kPairChunk;                 // [PC]
  float *l_s = m_s + kPairChunk;                     // [PC]
  unsigned long long *mask_s =
      reinterpret_cast<unsigned long long *>(l_s + 2 * kPairChunk);  // [PC]

  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int split = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int L, row0, R;
  if (!seq_shape(p, s, L, row0, R)) return;
  const int kb = split * p.keys_per_split;
  if (R == 0 || kb >= L) return;  // idle sequence or empty partition: skipped
  const int ke = min(kb + p.keys_per_split, L);
  const int C = L - R;
  const int G = p.group;
  const int P = G * R;
  const int row_bytes_head = D * kEsz;

  for (int pc0 = 0; pc0 < P; pc0 += kPairChunk) {
    const int npc = min(kPairChunk, P - pc0);
    // Q chunk, scaled by softmax_scale * log2(e) so scores are in log2 units
    for (int e = tid; e < kPairChunk * D; e += kThreads) {
      const int i = e / D, d = e - (e / D) * D;
      float v = 0.f;
      if (i < npc) {
        const int pr = pc0 + i, r = pr / G, h = g * G + (pr - r * G);
        v = p.q[((long long)(row0 + r) * p.n_q_heads + h) * D + d] * p.scale_log2;
      }
      Qs[e] = v;
    }
    if (tid < kPairChunk) {
      unsigned long long m = 0;
      if (tid < npc) {
        const int r = (pc0 + tid) / G;
        m = p.row_masks ? p.row_masks[row0 + r]
                        : (r >= 63 ? ~0ull : ((1ull << (r + 1)) - 1ull));
      }
      mask_s[tid] = m;
    }
    // this warp's pairs (warp + 4k) keep running max / sum in registers
    float m_run[kPairChunk / 4], l_run[kPairChunk / 4];
#pragma unroll
    for (int k = 0; k < kPairChunk / 4; ++k) {
      m_run[k] = -INFINITY;
      l_run[k] = 0.f;
    }
    const int dset = tid % Sh::kDimCover, pset = tid / Sh::kDimCover;
    float acc[Sh::kPairsPerThread][Sh::kDimsPerThread];
#pragma unroll
    for (int a = 0; a < Sh::kPairsPerThread; ++a)
#pragma unroll
      for (int b = 0; b < Sh::kDimsPerThread; ++b) acc[a][b] = 0.f;
    __syncthreads();

    for (int t0 = kb; t0 < ke; t0 += kTileKeys) {
      // load + convert this tile of K and V (one read per key row)
      for (int v = tid; v < kTileKeys * kVecPerRow; v += kThreads) {
        const int j = v / kVecPerRow, c = v - j * kVecPerRow;
        const int key = t0 + j;
        float kf[kElemPerVec], vf[kElemPerVec];
        bool ok = key < ke;
        const uint8_t *ka = nullptr, *va = nullptr;
        if (ok) {
          ka = kv_addr(p, p.k_pages, s, key, g, row_bytes_head);
          va = kv_addr(p, p.v_pages, s, key, g, row_bytes_head);
          ok = ka && va;
        }
        if (ok) {
          const uint4 kr = __ldg(reinterpret_cast<const uint4 *>(ka) + c);
          const uint4 vr = __ldg(reinterpret_cast<const uint4 *>(va) + c);
          Fmt::to_float(kr, kf);
          Fmt::to_float(vr, vf);
          if (p.scales) {
            // the stored vectors times their per-vector scales
            const float ks = kv_scale(p, p.k_pages, s, key, g);
            const float vs = kv_scale(p, p.v_pages, s, key, g);
#pragma unroll
            for (int e = 0; e < kElemPerVec; ++e) {
              kf[e] *= ks;
              vf[e] *= vs;
            }
          }
        } else {
#pragma unroll
          for (int e = 0; e < kElemPerVec; ++e) kf[e] = vf[e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < kElemPerVec; e += 4) {
          *reinterpret_cast<float4 *>(&Ks[j * Sh::kRow + c * kElemPerVec + e]) =
              make_float4(kf[e], kf[e + 1], kf[e + 2], kf[e + 3]);
          *reinterpret_cast<float4 *>(&Vs[j * Sh::kRow + c * kElemPerVec + e]) =
              make_float4(vf[e], vf[e + 1], vf[e + 2], vf[e + 3]);
        }
      }
      __syncthreads();

      // scores for key `lane` and pairs warp + 4k, then the online softmax
      {
        const int key = t0 + lane;
        float x[kPairChunk / 4];
#pragma unroll
        for (int k = 0; k < kPairChunk / 4; ++k) x[k] = 0.f;
        const float *krow = &Ks[lane * Sh::kRow];
#pragma unroll 4
        for (int d = 0; d < D; d += 4) {
          const float4 kv = *reinterpret_cast<const float4 *>(krow + d);
#pragma unroll
          for (int k = 0; k < kPairChunk / 4; ++k) {
            const float4 qv = *reinterpret_cast<const float4 *>(&Qs[(warp + 4 * k) * D + d]);
            x[k] = fmaf(qv.x, kv.x, x[k]);
            x[k] = fmaf(qv.y, kv.y, x[k]);
            x[k] = fmaf(qv.z, kv.z, x[k]);
            x[k] = fmaf(qv.w, kv.w, x[k]);
          }
        }
#pragma unroll
        for (int k = 0; k < kPairChunk / 4; ++k) {
          const int i = warp + 4 * k;
          const unsigned long long m = mask_s[i];
          const bool vis = i < npc && key < ke && (key < C || ((m >> (key - C)) & 1ull));
          const float xv = vis ? x[k] : -INFINITY;
          const float m_new = fmaxf(m_run[k], warp_max(xv));
          float pe = 0.f, alpha = 1.f;
          if (m_new != -INFINITY) {
            pe = vis ? exp2f(xv - m_new) : 0.f;
            alpha = exp2f(m_run[k] - m_new);  // 0 when nothing was seen yet
          }
          l_run[k] = l_run[k] * alpha + warp_sum(pe);
          m_run[k] = m_new;
          Ps[i * kTileKeys + lane] = pe;
          if (lane == 0) alpha_s[i] = alpha;
        }
      }
      __syncthreads();

      // O <- O * alpha + P . V for this thread's pairs and dims
#pragma unroll
      for (int a = 0; a < Sh::kPairsPerThread; ++a) {
        const float al = alpha_s[pset + Sh::kPairSets * a];
#pragma unroll
        for (int b = 0; b < Sh::kDimsPerThread; ++b) acc[a][b] *= al;
      }
      for (int j = 0; j < kTileKeys; j += 4) {
        float vv[4][Sh::kDimsPerThread];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
#pragma unroll
          for (int b = 0; b < Sh::kDimsPerThread; ++b)
            vv[jj][b] = Vs[(j + jj) * Sh::kRow + dset + b * Sh::kDimCover];
#pragma unroll
        for (int a = 0; a < Sh::kPairsPerThread; ++a) {
          const float4 pp =
              *reinterpret_cast<const float4 *>(&Ps[(pset + Sh::kPairSets * a) * kTileKeys + j]);
#pragma unroll
          for (int b = 0; b < Sh::kDimsPerThread; ++b) {
            acc[a][b] = fmaf(pp.x, vv[0][b], acc[a][b]);
            acc[a][b] = fmaf(pp.y, vv[1][b], acc[a][b]);
            acc[a][b] = fmaf(pp.z, vv[2][b], acc[a][b]);
            acc[a][b] = fmaf(pp.w, vv[3][b], acc[a][b]);
          }
        }
      }
      __syncthreads();
    }

    // partial results: o / l and lse (log2 units); -inf for no visible key
    if (lane == 0) {
#pragma unroll
      for (int k = 0; k < kPairChunk / 4; ++k) {
        m_s[warp + 4 * k] = m_run[k];
        l_s[warp + 4 * k] = l_run[k];
      }
    }
    __syncthreads();
#pragma unroll
    for (int a = 0; a < Sh::kPairsPerThread; ++a) {
      const int i = pset + Sh::kPairSets * a;
      if (i >= npc) continue;
      const int pr = pc0 + i, r = pr / G, h = g * G + (pr - r * G);
      const long long ph = ((long long)(row0 + r) * p.n_q_heads + h) * p.n_splits + split;
      const float l = l_s[i];
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
      for (int b = 0; b < Sh::kDimsPerThread; ++b)
        p.o_part[ph * D + dset + b * Sh::kDimCover] = acc[a][b] * inv;
      if (dset == 0) p.lse_part[ph] = l > 0.f ? m_s[i] + log2f(l) : -INFINITY;
    }
    __syncthreads();
  }
}

// ---- merge pass -------------------------------------------------------------

// 128-key tiles of sequence s as the tensor-core pass counts them.
__device__ __forceinline__ int seq_tiles_merge(const LseKernelParams &p, int s, int &L, int &row0,
                                               int &R) {
  L = p.seq_lens[s];
  row0 = p.row_offsets[s];
  R = p.row_offsets[s + 1] - row0;
  const long long cap = (long long)p.max_pages * p.tokens_per_fragment;
  if (row0 < 0 || R < 0 || R > p.max_rows || row0 + R > p.max_total_rows || R > L ||
      (long long)L > cap || R == 0)
    return 0;
  return (L + 127) / 128;
}

constexpr int kMergeWarps = 8;
constexpr int kMergeThreads = kMergeWarps * 32;

// One CTA (8 warps) per (row, query head) of the call's rows: blockIdx.x =
// row * Hq + head.  Before waiting for the partial pass the CTA finds the
// row's sequence and which partials of its segment are live (the scan over
// the sequences reads only call inputs, all threads at once, so it overlaps
// the partial pass's tail).  Each warp then loads its share of the partials
// (warp w: partials w, w + 8, ..., kUnroll in flight per lane, each lane a
// D/32 slice of the head dim) and keeps a running maximum of their lse; the
// warps' sums are rescaled to the common maximum and added in warp order in
// shared memory.
template <int D, int kUnroll>
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(
    const __grid_constant__ LseKernelParams p) {
  constexpr int kPerLane = D / 32;
  __shared__ float s_m[kMergeWarps], s_w[kMergeWarps];
  __shared__ float s_acc[kMergeWarps][D];
  __shared__ long long s_cnt[kMergeWarps][4];
  __shared__ int s_seq;
  const int h = blockIdx.x % p.n_q_heads;
  const int grow = blockIdx.x / p.n_q_heads;  // the row, over all sequences
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // the sequence holding the row: every thread tests its share of them
  if (tid == 0) s_seq = INT_MAX;
  __syncthreads();
  for (int q = tid; q < p.n_seqs; q += kMergeThreads)
    if (p.row_offsets[q] <= grow && grow < p.row_offsets[q + 1]) atomicMin(&s_seq, q);
  __syncthreads();
  const int s = s_seq;
  int L = 0, row0 = 0, R = 0;
  const bool live_row = s != INT_MAX && seq_shape(p, s, L, row0, R);
  const int r = grow - row0;  // row within the sequence
  int n_live = 0;
  if (p.balanced && live_row) {
    // pieces of the row's segment (sequence, row chunk, kv head) written by
    // the persistent tensor-core pass: the tiles of all segments end to end
    // (per sequence: row chunks x kv heads segments of its tiles), each
    // segment weighted by W more tiles, CTA c owning positions
    // [c UW / C, (c+1) UW / C); the tiles and segments before sequence s and
    // in all, summed over the CTA
    const int Rc = p.rows_per_chunk;
    long long mine_before = 0, mine_all = 0, segs_before = 0, segs_all = 0;
    for (int q = tid; q < p.n_seqs; q += kMergeThreads) {
      int Lq, r0q, Rq;
      const int n = seq_tiles_merge(p, q, Lq, r0q, Rq);
      const long long sq = n > 0 ? (long long)((Rq + Rc - 1) / Rc) * p.n_kv_heads : 0;
      const long long tq = (long long)n * sq;
      mine_all += tq;
      segs_all += sq;
      if (q < s) {
        mine_before += tq;
        segs_before += sq;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mine_before += __shfl_xor_sync(0xffffffffu, mine_before, o);
      mine_all += __shfl_xor_sync(0xffffffffu, mine_all, o);
      segs_before += __shfl_xor_sync(0xffffffffu, segs_before, o);
      segs_all += __shfl_xor_sync(0xffffffffu, segs_all, o);
    }
    if (lane == 0) {
      s_cnt[warp][0] = mine_before;
      s_cnt[warp][1] = mine_all;
      s_cnt[warp][2] = segs_before;
      s_cnt[warp][3] = segs_all;
    }
    __syncthreads();
    long long before = 0, U = 0, sb = 0, S = 0;
#pragma unroll
    for (int w = 0; w < kMergeWarps; ++w) {
      before += s_cnt[w][0];
      U += s_cnt[w][1];
      sb += s_cnt[w][2];
      S += s_cnt[w][3];
    }
    int Ls, r0s, Rs;
    const int n_s = seq_tiles_merge(p, s, Ls, r0s, Rs);
    const int g = h / p.group;
    const long long sid = sb + (long long)(r / Rc) * p.n_kv_heads + g;  // the segment
    const long long first = before + ((long long)(r / Rc) * p.n_kv_heads + g) * n_s;
    const long long C = U < p.n_ctas ? U : p.n_ctas;  // working CTAs of the partial pass
    const long long W =
        p.n_seqs <= kLseSeqTab && C > 0 && U / C >= kLseSegMinShare ? kLseSegWeight : 0;
    const long long UW = U + W * S;
    const long long pos0 = first + W * (sid + 1), pos1 = pos0 + n_s - 1;
    // one partial per piece
    n_live = n_s > 0 ? int(((pos1 + 1) * C - 1) / UW - ((pos0 + 1) * C - 1) / UW) + 1 : 0;
  } else if (live_row) {
    n_live = min((L + p.keys_per_split - 1) / p.keys_per_split, p.n_splits);
  }
  // partials are written by the preceding partial pass (programmatic launch)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (!live_row) return;  // uniform over the CTA
  const int row = grow;
  const long long base = ((long long)row * p.n_q_heads + h) * p.n_splits;
  const float *lse = p.lse_part + base;
  const float *o = p.o_part + base * D;

  // this warp's partials, kUnroll at a time, with a running maximum
  float m = -INFINITY, wsum = 0.f;
  float acc[kPerLane];
#pragma unroll
  for (int k = 0; k < kPerLane; ++k) acc[k] = 0.f;
  for (int i0 = warp; i0 < n_live; i0 += kMergeWarps * kUnroll) {
    float li[kUnroll], v[kUnroll][kPerLane];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int i = i0 + kMergeWarps * u;
      const bool in = i < n_live;
      li[u] = in ? lse[i] : -INFINITY;
#pragma unroll
      for (int k = 0; k < kPerLane; ++k)
        v[u][k] = in ? o[(long long)i * D + lane + 32 * k] : 0.f;
    }
    float mc = m;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) mc = fmaxf(mc, li[u]);
    if (mc == -INFINITY) continue;  // nothing live yet
    const float sc = exp2f(m - mc);  // 0 when m = -inf
    wsum *= sc;
#pragma unroll
    for (int k = 0; k < kPerLane; ++k) acc[k] *= sc;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const float w = li[u] == -INFINITY ? 0.f : exp2f(li[u] - mc);  // empty partial: 0
      wsum += w;
#pragma unroll
      for (int k = 0; k < kPerLane; ++k) acc[k] = fmaf(w, v[u][k], acc[k]);
    }
    m = mc;
  }
#pragma unroll
  for (int k = 0; k < kPerLane; ++k) s_acc[warp][lane + 32 * k] = acc[k];
  if (lane == 0) {
    s_m[warp] = m;
    s_w[warp] = wsum;
  }
  __syncthreads();
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kMergeWarps; ++w) M = fmaxf(M, s_m[w]);
  float scale[kMergeWarps];
  float wt = 0.f;
#pragma unroll
  for (int w = 0; w < kMergeWarps; ++w) {
    scale[w] = s_m[w] == -INFINITY ? 0.f : exp2f(s_m[w] - M);
    wt += s_w[w] * scale[w];
  }
  const float inv = wt > 0.f ? 1.f / wt : 0.f;
  float *out = p.out + ((long long)row * p.n_q_heads + h) * D;
  for (int d = tid; d < D; d += kMergeThreads) {
    float a = 0.f;
#pragma unroll
    for (int w = 0; w < kMergeWarps; ++w) a += s_acc[w][d] * scale[w];
    out[d] = a * inv;
  }
  if (p.lse_out && tid == 0)
    p.lse_out[(long long)row * p.n_q_heads + h] =
        wt > 0.f ? (M + log2f(wt)) * 0.69314718055994530942f : -INFINITY;
}

using lse_detail::SmemAllowed;
using lse_detail::allow_dynamic_smem;

template <int DT, int D>
int launch_cc(const LseKernelParams &p, int gx, int gy, int gz, int smem, cudaStream_t st) {
  auto k = partial_cuda_core_kernel<DT, D>;
  static SmemAllowed allowed;
  const int e = allow_dynamic_smem(k, smem, allowed);
  if (e) return e;
  k<<<dim3(gx, gy, gz), kThreads, smem, st>>>(p);
  return (int)cudaGetLastError();
}

template <int DT>
int launch_cc_d(const LseKernelParams &p, int D, int gx, int gy, int gz, int smem,
                cudaStream_t st) {
  switch (D) {
    case 64: return launch_cc<DT, 64>(p, gx, gy, gz, smem, st);
    case 128: return launch_cc<DT, 128>(p, gx, gy, gz, smem, st);
    case 256: return launch_cc<DT, 256>(p, gx, gy, gz, smem, st);
  }
  return (int)cudaErrorInvalidValue;
}

template <int DT, int D>
int occ_cc(int smem, int *n) {
  auto k = partial_cuda_core_kernel<DT, D>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return (int)e;
  return (int)cudaOccupancyMaxActiveBlocksPerMultiprocessor(n, k, kThreads, smem);
}

}  // namespace

int lse_partial_cuda_core_smem(int head_dim) {
  switch (head_dim) {
    case 64: return CcShape<64>::kSmemBytes;
    case 128: return CcShape<128>::kSmemBytes;
    case 256: return CcShape<256>::kSmemBytes;
  }
  return -1;
}

int lse_partial_cuda_core_occupancy(int dtype, int head_dim, int smem, int *n) {
  // occupancy depends on registers and shared memory, not on the format;
  // the BF16 instance stands for all
  (void)dtype;
  switch (head_dim) {
    case 64: return occ_cc<LSE_KV_BF16, 64>(smem, n);
    case 128: return occ_cc<LSE_KV_BF16, 128>(smem, n);
    case 256: return occ_cc<LSE_KV_BF16, 256>(smem, n);
  }
  return (int)cudaErrorInvalidValue;
}

int lse_launch_partial_cuda_core(const LseKernelParams &p, int dtype, int head_dim, int gx,
                                 int gy, int gz, int smem, void *stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  switch (dtype) {
    case LSE_KV_F32: return launch_cc_d<LSE_KV_F32>(p, head_dim, gx, gy, gz, smem, st);
    case LSE_KV_F16: return launch_cc_d<LSE_KV_F16>(p, head_dim, gx, gy, gz, smem, st);
    case LSE_KV_BF16: return launch_cc_d<LSE_KV_BF16>(p, head_dim, gx, gy, gz, smem, st);
    case LSE_KV_FP8_E4M3:
      return launch_cc_d<LSE_KV_FP8_E4M3>(p, head_dim, gx, gy, gz, smem, st);
    case LSE_KV_FP8_E5M2:
      return launch_cc_d<LSE_KV_FP8_E5M2>(p, head_dim, gx, gy, gz, smem, st);
  }
  return (int)cudaErrorInvalidValue;
}

// The merge is launched as a programmatic dependent of the partial pass on
// the same stream: its CTAs may be scheduled while the partial pass drains
// and wait in griddepcontrol.wait until the partial results are visible.
template <int D>
int launch_merge_d(const LseKernelParams &p, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  const long long grid = (long long)p.max_total_rows * p.n_q_heads;
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kMergeThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // With no more (row, head) CTAs than the partial pass had SMs, each CTA has
  // an SM to itself and merges up to 2 x SMs partials: it keeps 16 loads in
  // flight per lane (the round trips set its time).  Otherwise 8, which
  // leaves room for more resident CTAs.
  if (D <= 128 && p.balanced && grid <= p.n_ctas)
    return (int)cudaLaunchKernelEx(&cfg, merge_kernel<D, 16>, p);
  return (int)cudaLaunchKernelEx(&cfg, merge_kernel<D, 8>, p);
}

int lse_launch_merge(const LseKernelParams &p, int head_dim, void *stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  switch (head_dim) {
    case 64: return launch_merge_d<64>(p, st);
    case 128: return launch_merge_d<128>(p, st);
    case 256: return launch_merge_d<256>(p, st);
  }
  return (int)cudaErrorInvalidValue;
}

const char *lse_cuda_error_string(int code) { return cudaGetErrorString((cudaError_t)code); }
