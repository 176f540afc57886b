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
//    TMEM in FP32.  With 16-bit K/V, Q and P carry a hi + lo pair of 16-bit
//    terms (one term holds the value rounded to the storage's 16-bit format,
//    the other the rounding error) so the products keep ~16 mantissa bits
//    and only the K/V storage rounding remains.  With FP8 K/V the tiles
//    enter kind::f8f6f4 products as loaded: Q as four E4M3 terms under a
//    per-pair power-of-2 scale, P (times 2^7) as four E5M2 terms, each term
//    holding the rounding error of the ones before it.
//  * Softmax: two warpgroups take alternate tiles (ping-pong), each with
//    its own score buffer in TMEM, its own P tile in shared memory and its
//    own output accumulator, so one group's exponentials overlap the other
//    group's tensor-core work; each group writes its own partial result per
//    piece (the merge combines them like any other partials).  One thread
//    per key reads its row of S from TMEM.  The running maximum is rescaled
//    lazily: only when a score exceeds it by more than 2^8 are the maxima
//    recomputed and the group's TMEM output rescaled.
//  * K and V sit in separate rings, so a K slot is refilled as soon as its
//    score product is done.  A group's next score product waits only for
//    the group's softmax to finish reading its score buffer, and its next
//    softmax pass only for the output product that read its P tile.
//  * Each product issues one MMA per K step with all operand terms side by
//    side along N (an MMA costs its issuing thread the same whatever its
//    N), and the two products are issued by two threads; the row sums of P
//    are summed by the softmax warps.
//
// Roles: warp 0 TMA producer, warp 1 score-product issuer (and TMEM
// owner), warp 2 output-product issuer, warp 3 stages Q, then two to four
// softmax groups of four warps (128 threads, one per key of a tile), each
// taking an equal share of the tile's (row, head) pairs.
// Every wait is bounded: a wait that runs out sets LSE_DEVERR_TIMEOUT and
// every role leaves its loop; TMEM is released and outstanding copies are
// drained before the CTA exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cfloat>
#include <cstring>
#include <mutex>

#include "lse_internal.h"
#include "lse_smem_attr.h"
#include "lse_tc_ptx.h"

namespace {

using namespace lse_ptx;

constexpr int kTK = 128;           // keys per tile = M of the score product
constexpr int kD = 128;            // head dim = M of the output product
// Softmax groups per CTA for a pairs bucket: more groups give each thread
// fewer pairs of a tile (each group's share is a multiple of 4 pairs).
template <int P8>
constexpr int tc_groups() { return P8 == 48 || P8 == 24 ? 3 : 2; }
template <int P8>
constexpr int tc_threads() { return 128 * (1 + tc_groups<P8>()); }
constexpr float kTau = 8.f;        // lazy-rescale threshold (log2 units)
constexpr int kRegionBytes = kTK * 128;          // 128 rows x 128 B (64 dims)

struct __align__(64) TcParams {
  CUtensorMap maps[LSE_MAX_TMA_CHUNKS];
  LseKernelParams p;
  int n_ctas;
  int n_slots;
  int k_stages;  // K ring depth
  int v_stages;  // V ring depth (V tiles are held longer: through the softmax and P.V)
  int q_slots;
  int p_bufs;
  int box_tokens;
  int fused;  // 1: the merge runs in this pass and writes p.out / p.lse_out
  int withhold_tile;  // tests of the bounded waits: each CTA's tile of this index is not loaded
};

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

// Row chunks of a sequence: its R query rows are cut into chunks of at most
// rows_per_chunk rows (so a chunk's (row, head) pairs fit one score tile);
// each chunk reads all of the sequence's keys.
__device__ __forceinline__ int seq_chunks(const LseKernelParams &p, int R) {
  return (R + p.rows_per_chunk - 1) / p.rows_per_chunk;
}

// Per-sequence record built once per CTA in shared memory (sequences up to
// kSeqTab): tiles of all segments before the sequence, its 128-key tiles,
// L, first row, R, and the number of segments before the sequence.
constexpr int kSeqTab = kLseSeqTab;
struct SeqRec {
  int prefix, n_tiles, L, row0, R, seg_prefix;
};

// Walks the CTA's contiguous range of global tiles, segment by segment.  The
// segments of a sequence are (row chunk, kv head), chunk-major, each of
// n_tiles tiles.  With a sequence table it looks sequences up in shared
// memory; without one (more sequences than the table holds) it reads them
// from global memory.
struct TileIter {
  int s, c, g, tile, n_tiles;  // segment (sequence, row chunk, kv head), tile within it
  int n_chunks;
  int L, row0, R;              // the sequence
  int seg_id;                  // index of the segment among all segments of the call
  long long seg_first;         // global index of the segment's first tile
  long long t, t_end;          // current / end global tile
  const SeqRec *tab;           // shared-memory sequence table or null

  __device__ int tiles_of(const LseKernelParams &p, int q) {
    if (tab) {
      const SeqRec r = tab[q];
      L = r.L;
      row0 = r.row0;
      R = r.R;
      return r.n_tiles;
    }
    return seq_tiles(p, q, L, row0, R);
  }
  __device__ __forceinline__ void next_seq(const LseKernelParams &p) {
    // advance to the next sequence with tiles, starting at s
    while (s < p.n_seqs) {
      const int n = tiles_of(p, s);
      if (n > 0) {
        n_tiles = n;
        n_chunks = seq_chunks(p, R);
        return;
      }
      ++s;
    }
  }
  __device__ __forceinline__ void init(const LseKernelParams &p, long long t_begin,
                                       long long t_stop, const SeqRec *table) {
    t = t_begin;
    t_end = t_stop;
    tab = table;
    s = 0;
    long long base = 0;
    int seg_base = 0;
    n_tiles = 0;
    seg_id = 0;
    if (t >= t_end) return;
    if (tab) {
      // last sequence whose first tile is at or before t (idle sequences share
      // the prefix of the next one, so the last such index has tiles)
      int lo = 0, hi = p.n_seqs - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((long long)tab[mid].prefix <= t) lo = mid;
        else hi = mid - 1;
      }
      s = lo;
      base = tab[s].prefix;
      seg_base = tab[s].seg_prefix;
      next_seq(p);
    } else {
      next_seq(p);
      while (base + (long long)n_chunks * p.n_kv_heads * n_tiles <= t) {
        base += (long long)n_chunks * p.n_kv_heads * n_tiles;
        seg_base += n_chunks * p.n_kv_heads;
        ++s;
        next_seq(p);
      }
    }
    const int sg = int((t - base) / n_tiles);  // segment within the sequence
    c = sg / p.n_kv_heads;
    g = sg - c * p.n_kv_heads;
    tile = int((t - base) - (long long)sg * n_tiles);
    seg_first = base + (long long)sg * n_tiles;
    seg_id = seg_base + sg;
  }
  __device__ bool valid() const { return t < t_end; }
  __device__ bool seg_start(long long t_begin) const { return t == t_begin || tile == 0; }
  __device__ bool seg_end() const { return t == t_end - 1 || tile == n_tiles - 1; }
  // the segment's rows: global index of the first, count, and offset of the
  // first within the sequence
  __device__ int crow0(const LseKernelParams &p) const { return row0 + c * p.rows_per_chunk; }
  __device__ int crows(const LseKernelParams &p) const {
    return min(p.rows_per_chunk, R - c * p.rows_per_chunk);
  }
  __device__ void advance(const LseKernelParams &p) {
    ++t;
    if (t >= t_end) return;
    if (++tile == n_tiles) {
      tile = 0;
      seg_first += n_tiles;
      ++seg_id;
      if (++g == p.n_kv_heads) {
        g = 0;
        if (++c == n_chunks) {
          c = 0;
          ++s;
          next_seq(p);
        }
      }
    }
  }
};

// Cut of the live tiles into the working CTAs' ranges.  Every segment
// counts W tiles more than it has (the fixed cost of starting and ending
// one: its Q staged, its first tile's rescale, its epilogue), so a CTA whose
// range crosses many short segments gets fewer tiles.  Tile t of segment
// sid sits at position t + W (sid + 1) of UW = U + W S positions, and CTA c
// takes the tiles at positions [c UW / C, (c+1) UW / C).  W is 0 when the
// sequences are not in the shared-memory table, or when a CTA's share is
// under kSegMinShare tiles (there W would be a coarse share of a CTA's work;
// it also keeps every range non-empty).
constexpr int kSegWeight = kLseSegWeight;
constexpr int kSegMinShare = kLseSegMinShare;

// CTA whose range holds position x.
__device__ __forceinline__ int cta_of_pos(long long x, long long UW, int C) {
  return int(((x + 1) * (long long)C - 1) / UW);
}

// First tile at or after position x (U when x is past the last tile).
__device__ long long tile_at(const SeqRec *tab, int n_seqs, const LseKernelParams &p, int W,
                             long long U, long long UW, long long x) {
  if (x >= UW) return U;
  // last sequence whose weighted start is at or before x (an idle sequence
  // starts where the next one does, so the last such index has tiles)
  int lo = 0, hi = n_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((long long)tab[mid].prefix + (long long)W * tab[mid].seg_prefix <= x) lo = mid;
    else hi = mid - 1;
  }
  const SeqRec r = tab[lo];
  const long long o = x - ((long long)r.prefix + (long long)W * r.seg_prefix);
  const int nseg = seq_chunks(p, r.R) * p.n_kv_heads;
  const long long j = o / (r.n_tiles + W), k = o - j * (r.n_tiles + W);
  if (j >= nseg) return (long long)r.prefix + (long long)nseg * r.n_tiles;
  return (long long)r.prefix + j * r.n_tiles + (k > W ? k - W : 0);
}


// Fragment ids of the boxes of one tile (-1: past the sequence, -2: names
// no fragment, flagged).
__device__ __noinline__ void load_page_ids(const LseKernelParams &p, int seq, int tile, int L,
                                           int nbox, int box_t, int *pk, int *pv) {
  const int key0 = tile * kTK;
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

// TMA boxes of one tile (K or V): fragment ids ids[0..nbox), into dst.  A
// 16-bit tile is two regions of 64 dims (tensor rows 2g and 2g + 1); an
// FP8 tile is one region of 128 dims (tensor row g).
__device__ __forceinline__ void load_boxes(const TcParams &tp, int nbox, int box_t, int regions,
                                        int g, int key0, const int *ids, uint32_t dst,
                                        uint32_t full_bar) {
  const LseKernelParams &p = tp.p;
  const int T = p.tokens_per_fragment;
#pragma unroll 1
  for (int b = 0; b < nbox; ++b) {
    const int f = ids[b];
    if (f < 0) continue;
    const int kb = key0 + b * box_t;
    const int c = f / p.frags_per_chunk;
    const int z = (f - c * p.frags_per_chunk) * T + kb % T;
    const uint32_t d = dst + b * box_t * 128;
#pragma unroll 1
    for (int r = 0; r < regions; ++r)
      tma_load_3d(d + r * kRegionBytes, &tp.maps[c], full_bar, 0, g * regions + r, z);
  }
}

// Per-vector scales of one tile's boxes (kv head g) into a row of 128 FP32
// in shared memory: one bulk copy per box from entry (g, key % T) of the
// [kv_head][token] scale block of its fragment (fragment ids ids[0..nbox)).
__device__ __forceinline__ void load_scales(const LseKernelParams &p, int nbox, int box_t, int g,
                                            int key0, const int *ids, uint32_t dst,
                                            uint32_t full_bar) {
  const int T = p.tokens_per_fragment;
#pragma unroll 1
  for (int b = 0; b < nbox; ++b) {
    const int f = ids[b];
    if (f < 0) continue;
    const int kb = key0 + b * box_t;
    bulk_load(dst + (uint32_t)(b * box_t * 4),
              p.scales + ((long long)f * p.n_kv_heads + g) * T + kb % T, (uint32_t)box_t * 4u,
              full_bar);
  }
}

// Producer work for tile n: K slot, tile record, K boxes, V slot, V boxes
// (and, with sdst != 0, the tile's K and V scales into sdst[0..128) and
// sdst[128..256), counted on the V slot's barrier).  Returns 0 when a wait
// gave up.
__device__ __forceinline__ int produce_tile(const TcParams &tp, int n, int NK, int NV, int nbox,
                                            int box_t, int regions, int g, int tile, int L,
                                            const int *pk, const int *pv, uint32_t kdst,
                                            uint32_t vdst, uint32_t sdst, const uint32_t *bars_k,
                                            const uint32_t *bars_v, uint32_t info_bar,
                                            uint4 *info, volatile int *abort_flag) {
  const LseKernelParams &p = tp.p;
  const uint32_t ph_k = ((n / NK) & 1) ^ 1, ph_v = ((n / NV) & 1) ^ 1;
  const int key0 = tile * kTK;
  uint32_t kmask = 0, vmask = 0;
#pragma unroll 1
  for (int b = 0; b < nbox; ++b) {
    if (pk[b] >= 0) kmask |= 1u << b;
    if (pv[b] >= 0) vmask |= 1u << b;
  }
  const int live = L - key0 < kTK ? L - key0 : kTK;
  const uint32_t box_bytes = (uint32_t)regions * (uint32_t)box_t * 128u;
  if (!mbar_wait(bars_k[0], ph_k, abort_flag, p.err)) return 0;
  // the record slot was last read by the softmax of tile n - 8, which has
  // finished: the K slot of tile n was freed by the score product of tile
  // n - NK, issued in order after the softmax of tiles up to n - NK - 2
  // (>= n - 8 for NK <= 6) read their scores
  *info = make_uint4(kmask, vmask, (uint32_t)live, 0u);
  mbar_arrive(info_bar);  // publishes the record
  mbar_expect_tx(bars_k[1], (uint32_t)__popc(kmask) * box_bytes);
  load_boxes(tp, nbox, box_t, regions, g, key0, pk, kdst, bars_k[1]);
  if (!mbar_wait(bars_v[0], ph_v, abort_flag, p.err)) return 0;
  const uint32_t scale_bytes =
      sdst ? (uint32_t)(__popc(kmask) + __popc(vmask)) * (uint32_t)box_t * 4u : 0u;
  mbar_expect_tx(bars_v[1], (uint32_t)__popc(vmask) * box_bytes + scale_bytes);
  load_boxes(tp, nbox, box_t, regions, g, key0, pv, vdst, bars_v[1]);
  if (sdst) {
    load_scales(p, nbox, box_t, g, key0, pk, sdst, bars_v[1]);
    load_scales(p, nbox, box_t, g, key0, pv, sdst + kTK * 4, bars_v[1]);
  }
  return 1;
}


// A segment this CTA shares with other CTAs, merged after the CTA's own
// tiles when the merge is fused into the pass (at most two per CTA: the
// first and the last segment of its range; every segment in between lies
// in this CTA alone).
struct EndRec {
  int seg_id, n_pieces, piece, row0, rows, g;
};
// shared memory of the end phase: a flag word pair, up to two end records
// and their count; then the CTA's tile range {t_begin, t_stop, UW, W}
constexpr int kEndBytes = 2 * 4 + 2 * (int)sizeof(EndRec) + 8 + 8 + 4 * 8;

// ---- shared-memory and TMEM layout ------------------------------------------------

constexpr bool is_f8(int dt) { return dt == LSE_KV_FP8_E4M3 || dt == LSE_KV_FP8_E5M2; }

// FP8 operands: Q and P enter the 8-bit products as sums of kTerms 8-bit
// values (each term holds the rounding error of the ones before it).
constexpr int kQTerms = 4;         // E4M3 terms of Q (per-pair power-of-2 scale)
constexpr int kPTerms = 4;         // E5M2 terms of P
constexpr int kPScaleLog2 = 7;     // P enters the FP8 products times 2^7

template <int DT, int P8>
struct TcLayout {
  static constexpr bool kF8 = is_f8(DT);
  static constexpr int kNQ = (P8 + 15) / 16 * 16;       // pairs rounded to 16 (MMA N step)
  // each softmax group takes an equal share of the (row, head) pairs of
  // every tile
  static constexpr int kG = tc_groups<P8>();
  static constexpr int kH = P8 / kG;
  static_assert(kH % 4 == 0, "a group's pairs come in blocks of 4");
  // Every product carries its operand terms side by side along N, so one
  // MMA per K step covers them all (the issue of an MMA costs the same
  // whatever its N).  Score columns of a tile: 16-bit, Q hi | Q lo blocks of
  // kNQ; FP8, four Q-term blocks of kNQ.
  static constexpr int kSW = kF8 ? kQTerms * kNQ : 2 * kNQ;
  // Output columns of a slot: 16-bit, P hi | P lo blocks of P8; FP8, four
  // P-term blocks of kNQ when they fit in TMEM, else one block that the
  // four terms accumulate into (four MMAs per K step)
  static constexpr bool kPSide = !kF8 || 2 * kSW + kPTerms * kNQ <= 512;
  static constexpr int kOBlk = kF8 ? kNQ : P8;            // width of one output block
  static constexpr int kN = kF8 ? (kPSide ? kPTerms * kNQ : kNQ) : 2 * P8;
  static constexpr int kQRegion = kNQ * 128;             // kNQ rows of 128 bytes
  // 16-bit: two 64-dim regions, each [hi rows | lo rows]; FP8: one 128-dim
  // region of kQTerms x kNQ rows
  static constexpr int kQBytes = 4 * kQRegion;
  static_assert(!kF8 || kQTerms == 4, "Q slot holds four FP8 terms");
  // P^T operand, MN-major without swizzle: core matrices of 8 keys x 16
  // bytes (8 16-bit or 16 FP8 columns); 8-key groups kPLbo apart; columns
  // hi block then lo block (16-bit) or term blocks of kNQ (FP8)
  static constexpr int kPCols = kF8 ? kPTerms * kNQ : 2 * P8;
  static constexpr int kPLbo = (kF8 ? kPCols / 16 : kPCols / 8) * 128;
  static constexpr int kPBytes = kTK / 8 * kPLbo;        // one tile's P
  // TMEM: two score buffers (tiles alternate), then the output slots (two
  // when they fit: a piece's output is read out while the next one builds)
  static constexpr int kOSlots = (2 * kSW + 2 * kN <= 512) ? 2 : 1;
  static constexpr int kTmemNeed = 2 * kSW + kOSlots * kN;
  static constexpr int kTmemCols = kTmemNeed <= 64 ? 64 : kTmemNeed <= 128 ? 128
                                 : kTmemNeed <= 256 ? 256 : 512;
  static_assert(kTmemNeed <= 512, "TMEM holds at most 512 columns");
  static_assert(kSW <= 256 && kN <= 256, "MMA N is at most 256");
  static constexpr int kBars = 64;
  static constexpr int kMiscBytes = kBars * 8 + 16 + kG * 64 * 4 * 2 + kG * 4 * 64 * 4 +
                                    kG * 64 * 8 * 2 + 64 * 4 + 8 * 16 + 2 * 32 * 16 * 4 +
                                    (kF8 ? (2 + kG) * 64 * 4 : 0) +
                                    kSeqTab * (int)sizeof(SeqRec) + kEndBytes;
  // one K or V tile: 128 keys of 128 dims (two 64-dim regions when 16-bit)
  static constexpr int kHalfStage = kF8 ? kRegionBytes : 2 * kRegionBytes;
  // per-vector scales of one tile, K then V (128 FP32 each), per ring stage
  static constexpr int kScStage = 2 * kTK * 4;
  // k_stages / v_stages: K and V ring depths; q_slots: Q ring depth (1 or
  // 2); p_bufs: P tiles (1 or 2); scaled: per-vector scale rows per V stage
  static int smem_bytes(int k_stages, int v_stages, int q_slots, int p_bufs, bool scaled) {
    return 1024 + (k_stages + v_stages) * kHalfStage + q_slots * kQBytes + p_bufs * kPBytes +
           (scaled ? v_stages * kScStage : 0) + kMiscBytes;
  }
};

// barrier indices in the misc block
constexpr int kMaxStages = 6;  // K/V ring depth limit (tile records: ring of 8)
enum {
  kBarFullK = 0,    // [8]
  kBarEmptyK = 8,   // [8]
  kBarFullV = 16,   // [8]
  kBarEmptyV = 24,  // [8]
  kBarSFull = 32,   // [2] per score buffer: its product is complete
  kBarPFull = 34,   // [2] per P tile: every group wrote its probabilities
  kBarQFull = 36,   // [2]
  kBarQEmpty = 38,  // [2]
  kBarOFull = 40,   // [2] per output slot: the piece's last output product is complete
  kBarOEmpty = 42,  // [2] per output slot: every group read it out
  kBarDone = 44,    // the score issuer's MMAs have completed
  kBarInfo = 45,    // [8] one per tile record
  kBarPEmpty = 53,  // [2] per P tile: the output product that read it is complete
  kBarDoneV = 55,   // the output issuer's MMAs have completed
  kBarSEmpty = 56,  // [2] per score buffer: every group read it out
};

// Stage one segment's Q into a Q slot, by T threads (t = 0 .. T-1): each
// (pair row n, 8-dim chunk c) item is scaled by the softmax scale (log2
// units) and written in the operand layout of the score product.  Item
// t + T k goes to thread t, so the 16 lanes of a half warp hold one row.
// Items go in rounds of up to 8 per thread; the first round's loads, and L2
// prefetches of the later rounds' rows, are issued before `before_store` (the
// wait for the slot) runs.  FP8: each row
// is scaled by 2^e (max |x| 2^e in [128, 256)) and written as kQTerms E4M3
// terms; 2^-e goes to isig[n].
template <int DT, int P8, int T, class Wait>
__device__ __forceinline__ bool stage_q(const LseKernelParams &p, int t, int g, int row0, int P,
                                        uint8_t *qs, float *isig, Wait before_store) {
  using Lay = TcLayout<DT, P8>;
  constexpr int kNQ = Lay::kNQ;
  constexpr int kItems = kNQ * 16 / T;
  constexpr int kRound = kItems < 8 ? kItems : 8;
  static_assert(kItems * T == kNQ * 16, "items split evenly");
  const int G = p.group;
  const float sc = p.scale_log2;
  auto src_of = [&](int n, int c) {
    const int r = n / G, h = g * G + (n - r * G);
    return reinterpret_cast<const float4 *>(p.q + ((long long)(row0 + r) * p.n_q_heads + h) * kD +
                                            c * 8);
  };
  // the later rounds' rows into L2 (one prefetch per 128-byte line)
#pragma unroll 1
  for (int k = kRound; k < kItems; ++k) {
    const int item = t + T * k;
    const int n = item >> 4, c = item & 15;
    if (n < P && (c & 3) == 0)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(src_of(n, c)) : "memory");
  }
#pragma unroll 1
  for (int r0 = 0; r0 < kItems; r0 += kRound) {
    float4 ld[kRound][2];
#pragma unroll
    for (int k = 0; k < kRound; ++k) {
      const int item = t + T * (r0 + k);
      const int n = item >> 4, c = item & 15;
      if (n < P) {
        const float4 *src = src_of(n, c);
        ld[k][0] = __ldg(src);
        ld[k][1] = __ldg(src + 1);
      } else {
        ld[k][0] = ld[k][1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    if (r0 == 0 && !before_store()) return false;
#pragma unroll
    for (int k = 0; k < kRound; ++k) {
      const int item = t + T * (r0 + k);
      const int n = item >> 4, c = item & 15;
      float x[8] = {ld[k][0].x * sc, ld[k][0].y * sc, ld[k][0].z * sc, ld[k][0].w * sc,
                    ld[k][1].x * sc, ld[k][1].y * sc, ld[k][1].z * sc, ld[k][1].w * sc};
      if constexpr (Lay::kF8) {
        float mx = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(x[i]));
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        int e = 0;
        if (mx > 0.f && mx <= FLT_MAX) {
          const int E = ((__float_as_int(mx) >> 23) & 0xff) - 127;
          e = min(max(7 - E, -126), 126);
        }
        const float sg = exp2i(e);
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] *= sg;
        uint2 w[kQTerms];
        f8_terms<false, kQTerms>(x, w);
        // one 128-byte swizzled row per term
        const uint32_t off =
            (n >> 3) * 1024 + (n & 7) * 128 + ((((c >> 1) ^ (n & 7))) << 4) + (c & 1) * 8;
#pragma unroll
        for (int tt = 0; tt < kQTerms; ++tt)
          *reinterpret_cast<uint2 *>(qs + tt * Lay::kQRegion + off) = w[tt];
        if (c == 0) isig[n] = exp2i(-e);
      } else {
        uint4 vh, vl;
        split2<DT>(x[0], x[1], vh.x, vl.x);
        split2<DT>(x[2], x[3], vh.y, vl.y);
        split2<DT>(x[4], x[5], vh.z, vl.z);
        split2<DT>(x[6], x[7], vh.w, vl.w);
        // region (64 dims) of 2 kNQ rows: hi rows, then lo rows
        const int region = c >> 3, cc = c & 7;
        const uint32_t off = region * 2 * Lay::kQRegion + (n >> 3) * 1024 + (n & 7) * 128 +
                             ((cc ^ (n & 7)) << 4);
        *reinterpret_cast<uint4 *>(qs + off) = vh;
        *reinterpret_cast<uint4 *>(qs + Lay::kQRegion + off) = vl;
      }
    }
  }
  fence_proxy_async();  // the score product reads Q through the async proxy
  return true;
}

// L2 prefetch of one segment's Q: `rows` rows from row0, the G heads of kv
// head g (G x 512 contiguous bytes per row), by the 32 lanes of a warp.
__device__ __forceinline__ void prefetch_q(const LseKernelParams &p, int g, int row0, int rows,
                                           int lane) {
  const int G = p.group;
  const int lines = G * 4;  // 128-byte lines per row
  for (int i = lane; i < rows * lines; i += 32) {
    const int r = i / lines, l = i - r * lines;
    const float *a = p.q + ((long long)(row0 + r) * p.n_q_heads + g * G) * kD + l * 32;
    asm volatile("prefetch.global.L2 [%0];" ::"l"(a) : "memory");
  }
}

// End phase of the fused pass: for each segment this CTA shares with other
// CTAs, wait until every piece's partial is written (the segment's arrival
// count reaches kArrivals per piece: one per softmax group), then merge this
// CTA's share of the segment's (row, head) pairs: pair q goes to the
// segment's piece q mod n,
// so the n CTAs of the segment split its pairs.  A pair is merged by one or
// more warps, each taking every k-th piece with its loads issued together
// (lanes over the head dim, four dims a lane) and a running maximum; the
// warps' sums meet in shared memory (the K/V ring, idle by now).  Same
// arithmetic as the separate merge pass: M = max lse, weights 2^(lse - M).
// The last CTA to finish a segment clears its two counters for the next
// call.  The wait is bounded like every other wait; the launch is
// cooperative, so every CTA of the grid is resident and each arrives for its
// own pieces without waiting on any other CTA.
template <int kWarps, int kArrivals>
__device__ __noinline__ void fused_end_merge(const TcParams &tp, const EndRec *rec, int n_rec,
                                             volatile int *abort_flag, int *go_flag,
                                             float *scratch) {
  const LseKernelParams &p = tp.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float *w_m = scratch;                 // [warp] running maximum
  float *w_l = scratch + kWarps;        // [warp] sum of weights
  float *w_acc = scratch + 2 * kWarps;  // [warp][kD] weighted sums
#pragma unroll 1
  for (int k = 0; k < n_rec; ++k) {
    const EndRec r = rec[k];
    unsigned int *cnt = p.seg_count + 2 * r.seg_id;
    if (tid == 0) {
      int go = *abort_flag == 0;
      const long long t0 = clock64();
      while (go) {
        unsigned int v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(cnt) : "memory");
        if (v >= (unsigned)kArrivals * (unsigned)r.n_pieces) break;
        if (clock64() - t0 > kWaitCycles) {
          *abort_flag = 1;
          atomicOr(p.err, LSE_DEVERR_TIMEOUT);
          go = 0;
        }
        __nanosleep(64);
      }
      *go_flag = go;
    }
    __syncthreads();
    const bool go = *go_flag != 0;
    const int G = p.group, P = G * r.rows, n = r.n_pieces;
    // this CTA's pairs: r.piece, r.piece + n, ...
    const int mine = r.piece < P ? (P - 1 - r.piece) / n + 1 : 0;
#pragma unroll 1
    for (int b = 0; go && b < mine; b += kWarps) {
      const int np = min(kWarps, mine - b);           // pairs in this batch
      const int kw = kWarps / np;                      // warps per pair
      const int slot = warp / kw, sub = warp - slot * kw;
      const bool active = slot < np;
      float m = -INFINITY, l = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      long long base = 0;
      if (active) {
        const int q = r.piece + (b + slot) * n;
        const int rr = q / G, h = r.g * G + (q - rr * G);
        const long long oi = (long long)(r.row0 + rr) * p.n_q_heads + h;
        base = oi * tp.n_slots;
        // pieces sub, sub + kw, ...: loads first, then the running maximum
#pragma unroll 1
        for (int i0 = sub; i0 < n; i0 += 8 * kw) {
          float li[8];
          float4 vi[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * kw;
            li[u] = i < n ? __ldcg(p.lse_part + base + i) : -INFINITY;
            vi[u] = i < n ? __ldcg(reinterpret_cast<const float4 *>(p.o_part + (base + i) * kD) +
                                   lane)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
          }
          float mc = m;
#pragma unroll
          for (int u = 0; u < 8; ++u) mc = fmaxf(mc, li[u]);
          if (mc == -INFINITY) continue;
          const float sc = ex2(m - mc);  // 0 while m = -inf
          l *= sc;
          acc.x *= sc; acc.y *= sc; acc.z *= sc; acc.w *= sc;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float w = li[u] == -INFINITY ? 0.f : ex2(li[u] - mc);
            l += w;
            acc.x = fmaf(w, vi[u].x, acc.x);
            acc.y = fmaf(w, vi[u].y, acc.y);
            acc.z = fmaf(w, vi[u].z, acc.z);
            acc.w = fmaf(w, vi[u].w, acc.w);
          }
          m = mc;
        }
      }
      if (lane == 0) {
        w_m[warp] = m;
        w_l[warp] = l;
      }
      reinterpret_cast<float4 *>(w_acc + warp * kD)[lane] = acc;
      __syncthreads();
      // the pair's warps combined in a fixed order (warp `slot * kw` writes)
      if (active && sub == 0) {
        float M = -INFINITY;
        for (int s2 = 0; s2 < kw; ++s2) M = fmaxf(M, w_m[warp + s2]);
        float W = 0.f;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s2 = 0; s2 < kw; ++s2) {
          const float sc = w_m[warp + s2] == -INFINITY ? 0.f : ex2(w_m[warp + s2] - M);
          W += w_l[warp + s2] * sc;
          const float4 v = reinterpret_cast<const float4 *>(w_acc + (warp + s2) * kD)[lane];
          a.x = fmaf(sc, v.x, a.x);
          a.y = fmaf(sc, v.y, a.y);
          a.z = fmaf(sc, v.z, a.z);
          a.w = fmaf(sc, v.w, a.w);
        }
        const float inv = W > 0.f ? rcp(W) : 0.f;
        const long long oi = base / tp.n_slots;
        reinterpret_cast<float4 *>(p.out + oi * kD)[lane] =
            make_float4(a.x * inv, a.y * inv, a.z * inv, a.w * inv);
        if (lane == 0 && p.lse_out)
          p.lse_out[oi] = W > 0.f ? (M + lg2(W)) * 0.69314718055994530942f : -INFINITY;
      }
      __syncthreads();
    }
    __syncthreads();
    if (tid == 0 && go) {
      // leaving the segment: the last CTA out clears its counters
      const unsigned int left = atomicAdd(cnt + 1, 1u);
      if (left + 1u == (unsigned)r.n_pieces) {
        atomicExch(cnt, 0u);
        atomicExch(cnt + 1, 0u);
      }
    }
  }
}

template <int DT, int P8, bool kSc>
__global__ void __launch_bounds__(tc_threads<P8>(), 1)
    partial_tcgen05_kernel(const __grid_constant__ TcParams tp) {
  using Lay = TcLayout<DT, P8>;
  constexpr bool kF8 = Lay::kF8;
  constexpr int kG = Lay::kG;                    // softmax groups
  constexpr int kThreads = tc_threads<P8>();
  static_assert(!kSc || kF8, "per-vector scales go with the 8-bit formats");
  constexpr bool kE5 = DT == LSE_KV_FP8_E5M2;
  constexpr int kNQ = Lay::kNQ;
  constexpr int kN = Lay::kN;
  const int QS = tp.q_slots;
  const int PB = tp.p_bufs;
  const LseKernelParams &p = tp.p;
  const int NK = tp.k_stages, NV = tp.v_stages;
  const int cta = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t k_base = sbase;                                // K ring
  const uint32_t v_base = k_base + NK * Lay::kHalfStage;        // V ring
  const uint32_t q_base = v_base + NV * Lay::kHalfStage;        // Q slots
  const uint32_t p_base = q_base + QS * Lay::kQBytes;          // P tiles [buffer]
  const uint32_t sc_base = p_base + PB * Lay::kPBytes;         // scale rows [stage]
  uint8_t *misc = smem + (sc_base - sbase) + (kSc ? NV * Lay::kScStage : 0);
  // the P tile of tile n
  auto p_tile = [&](int n) { return p_base + (uint32_t)((n % PB) * Lay::kPBytes); };
  uint64_t *bars = reinterpret_cast<uint64_t *>(misc);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + Lay::kBars * 8);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + Lay::kBars * 8 + 4);
  long long *shared_u = reinterpret_cast<long long *>(misc + Lay::kBars * 8 + 8);
  float *m_run_all = reinterpret_cast<float *>(misc + Lay::kBars * 8 + 16);  // [kG][64]
  float *alpha_all = m_run_all + kG * 64;                                    // [kG][64]
  float *red_all = alpha_all + kG * 64;                                      // [kG][4][64]
  unsigned long long *masks_all =
      reinterpret_cast<unsigned long long *>(red_all + kG * 4 * 64);         // [kG][64]
  // per softmax group and draft key k of the sequence: the pairs that see it
  unsigned long long *visk_all = masks_all + kG * 64;                        // [kG][64]
  int *pair_row = reinterpret_cast<int *>(visk_all + kG * 64);               // [64]
  // ring of 8 per-tile records written by the producer before its arrival on
  // the tile's K barrier: {K box mask, V box mask, keys of the tile below L}
  uint4 *tile_info = reinterpret_cast<uint4 *>(pair_row + 64);               // [8]
  // fragment ids of a batch of 32 tiles (up to 16 boxes each), K then V
  int *page_buf = reinterpret_cast<int *>(tile_info + 8);                    // [2][32][16]
  // FP8: the inverse of Q's per-pair scale, per Q slot [0, 2) and the
  // copy each softmax group keeps for its segment [2, 2 + kG)
  float *isig_all = reinterpret_cast<float *>(page_buf + 2 * 32 * 16);       // [2+kG][64]
  SeqRec *seq_tab =
      reinterpret_cast<SeqRec *>(isig_all + (kF8 ? (2 + kG) * 64 : 0));     // [kSeqTab]
  int *had_all = reinterpret_cast<int *>(seq_tab + kSeqTab);                 // [2] (end phase)
  EndRec *end_rec = reinterpret_cast<EndRec *>(had_all + 2);                 // [2]
  int *n_end = reinterpret_cast<int *>(end_rec + 2);
  long long *range = reinterpret_cast<long long *>(
      (reinterpret_cast<uintptr_t>(n_end + 1) + 7) & ~uintptr_t(7));  // [4]
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  // the merge pass may be scheduled now; it waits for this grid to finish
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // ---- prologue: TMEM, total live tiles, barriers --------------------------------
  if (warp == 1) {
    // allocated first, while warp 0 reads the sequences' lengths
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(Lay::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  const bool use_tab = p.n_seqs <= kSeqTab;
  if (warp == 0) {
    // the barriers first (the producer uses them as soon as its table is
    // built, without waiting for the other warps)
    if (lane == 0) {
    *abort_flag = 0;
    for (int i = 0; i < 8; ++i) {
      mbar_init(bar(kBarFullK + i), 1);
      mbar_init(bar(kBarEmptyK + i), 1);
      mbar_init(bar(kBarFullV + i), 1);
      mbar_init(bar(kBarEmptyV + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kBarOFull + i), 1);
      mbar_init(bar(kBarOEmpty + i), 128 * kG);  // every group read its pairs out
    }
    *n_end = 0;
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kBarSFull + i), 1);
      mbar_init(bar(kBarSEmpty + i), 128 * kG);  // every group read its columns
      mbar_init(bar(kBarPFull + i), 128 * kG);   // every group wrote its columns
      mbar_init(bar(kBarQFull + i), 1);
      // FP8: the softmax groups also hold the slot until they have copied
      // the segment's Q scales
      mbar_init(bar(kBarQEmpty + i), kF8 ? 1 + kG : 1);
    }
    mbar_init(bar(kBarDone), 1);
    mbar_init(bar(kBarDoneV), 1);
    for (int i = 0; i < 8; ++i) mbar_init(bar(kBarInfo + i), 1);
    for (int i = 0; i < 2; ++i) mbar_init(bar(kBarPEmpty + i), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
      }
    __syncwarp();
    // every sequence's tiles, lanes taking contiguous blocks; then a warp
    // exclusive scan gives each sequence its first tile
    const int per = (p.n_seqs + 31) / 32;
    const int s0 = lane * per, s1 = min(p.n_seqs, s0 + per);
    long long mine = 0;
    bool bad = false;
    for (int q = s0; q < s1; ++q) {
      int L, r0, R;
      int n = seq_tiles(p, q, L, r0, R);
      if (n < 0) {
        bad = true;
        n = 0;
      }
      if (use_tab) seq_tab[q] = SeqRec{0, n, L, r0, R, 0};
      // all segments of the sequence: row chunks x kv heads
      mine += (long long)n * (n > 0 ? seq_chunks(p, R) : 0) * p.n_kv_heads;
    }
    long long incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int seg_total = 0;  // segments up to this lane's sequences (with the table)
    if (use_tab) {
      // segments of the lanes before this one (a second warp scan)
      int segs = 0;
      for (int q = s0; q < s1; ++q) {
        const int n = seq_tab[q].n_tiles;
        segs += n > 0 ? seq_chunks(p, seq_tab[q].R) * p.n_kv_heads : 0;
      }
      int seg_incl = segs;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, seg_incl, o);
        if (lane >= o) seg_incl += v;
      }
      seg_total = seg_incl;
      long long run = incl - mine;
      int seg_run = seg_incl - segs;
      for (int q = s0; q < s1; ++q) {
        seq_tab[q].prefix = (int)run;
        seq_tab[q].seg_prefix = seg_run;
        const int n = seq_tab[q].n_tiles;
        run += (long long)n * (n > 0 ? seq_chunks(p, seq_tab[q].R) : 0) * p.n_kv_heads;
        seg_run += n > 0 ? seq_chunks(p, seq_tab[q].R) * p.n_kv_heads : 0;
      }
    }
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 31) *shared_u = incl;
    if (lane == 0 && bad && cta == 0) atomicOr(p.err, LSE_DEVERR_BAD_LENGTH);
    // this CTA's range of tiles
    const long long U0 = __shfl_sync(0xffffffffu, incl, 31);
    const int S0 = use_tab ? __shfl_sync(0xffffffffu, seg_total, 31) : 0;
    if (lane == 0 && U0 > 0) {
      const int C0 = (int)(U0 < tp.n_ctas ? U0 : tp.n_ctas);
      const int W = use_tab && U0 / C0 >= kSegMinShare ? kSegWeight : 0;
      const long long UW = U0 + (long long)W * S0;
      long long b0 = UW * cta / C0, b1 = UW * (cta + 1) / C0;
      if (W > 0) {
        b0 = tile_at(seq_tab, p.n_seqs, p, W, U0, UW, b0);
        b1 = tile_at(seq_tab, p.n_seqs, p, W, U0, UW, b1);
      }
      range[0] = b0;
      range[1] = b1;
      range[2] = UW;
      range[3] = W;
    }
  }
  const SeqRec *tab = use_tab ? seq_tab : nullptr;
  if (tid < 64) pair_row[tid] = tid / p.group;
  // The other warps wait for warp 0's table, barriers and TMEM address;
  // warp 0 only announces its part (bar.arrive) and goes on to the loads.
  if (warp == 0) {
    asm volatile("bar.arrive 15, %0;" ::"n"(kThreads) : "memory");
  } else {
    tc_fence_before();
    asm volatile("bar.sync 15, %0;" ::"n"(kThreads) : "memory");
    tc_fence_after();
  }
  __syncwarp();
  const uint32_t tmem = warp == 0 ? 0u : *tmem_slot;  // (warp 0 never touches TMEM)
  const long long U = *shared_u;
  // working CTAs: never more than tiles, so no working range is empty and a
  // segment's pieces never outnumber its tiles
  const int C = (int)(U < tp.n_ctas ? U : tp.n_ctas);
  if (cta >= C) {  // nothing for this CTA (uniform): give the TMEM back
    if (warp == 1)
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                   "r"(Lay::kTmemCols)
                   : "memory");
    return;
  }
  const long long t_begin = range[0], t_stop = range[1], UW = range[2];
  const int W = (int)range[3];
  constexpr int kSW = Lay::kSW;
  // score buffer of tile n: n & 1; output slot of the CTA's segment seg: seg % kOS
  auto tmem_s = [&](int buf) { return tmem + (uint32_t)(buf * kSW); };
  constexpr int kOS = Lay::kOSlots;
  auto tmem_o = [&](int slot) { return tmem + (uint32_t)(2 * kSW + slot * kN); };

  const int box_t = tp.box_tokens;
  const int nbox = box_t >= kTK ? 1 : kTK / box_t;
  const uint32_t full_boxes = nbox >= 32 ? 0xffffffffu : ((1u << nbox) - 1u);
  const int G = p.group;

  if (warp == 0) {
    // ============================ TMA producer ============================
    // The warp reads the fragment ids of 32 tiles at once (one lane per
    // tile), then lane 0 streams the tiles: K then V of each, each into its
    // ring.
    const int n_total = (int)(t_stop - t_begin);
    int *pk = page_buf, *pv = page_buf + 32 * 16;
    int n = 0;
    bool ok = true;
#pragma unroll 1
    for (int b0 = 0; b0 < n_total && ok; b0 += 32) {
      const int cnt = n_total - b0 < 32 ? n_total - b0 : 32;
      TileIter mine;
      mine.init(p, t_begin + b0 + (lane < cnt ? lane : 0), t_stop, tab);
      if (lane < cnt)
        load_page_ids(p, mine.s, mine.tile, mine.L, nbox, box_t, pk + lane * 16, pv + lane * 16);
      __syncwarp();
#pragma unroll 1
      for (int i = 0; i < cnt; ++i, ++n) {
        const int tg = __shfl_sync(0xffffffffu, mine.g, i);
        const int tt = __shfl_sync(0xffffffffu, mine.tile, i);
        const int tl = __shfl_sync(0xffffffffu, mine.L, i);
        int go = 1;
        if (lane == 0 && n != tp.withhold_tile) {
          const uint32_t bars_k[2] = {bar(kBarEmptyK + n % NK), bar(kBarFullK + n % NK)};
          const uint32_t bars_v[2] = {bar(kBarEmptyV + n % NV), bar(kBarFullV + n % NV)};
          go = produce_tile(tp, n, NK, NV, nbox, box_t, kF8 ? 1 : 2, tg, tt, tl, pk + i * 16,
                            pv + i * 16,
                            k_base + (n % NK) * Lay::kHalfStage,
                            v_base + (n % NV) * Lay::kHalfStage,
                            kSc ? sc_base + (n % NV) * Lay::kScStage : 0u, bars_k, bars_v,
                            bar(kBarInfo + (n & 7)), tile_info + (n & 7), abort_flag);
        }
        go = __shfl_sync(0xffffffffu, go, 0);
        if (!go) {
          ok = false;
          break;
        }
      }
      __syncwarp();
    }
    // drain: every copy issued must have landed before the CTA exits
    if (lane == 0)
#pragma unroll 1
      for (int k = (n > NV ? n - NV : 0); k < n; ++k) {
        if (k >= n - NK) mbar_drain(bar(kBarFullK + k % NK), (k / NK) & 1);
        mbar_drain(bar(kBarFullV + k % NV), (k / NV) & 1);
      }
  } else if (warp == 1 || warp == 2) {
    // ====================== MMA issuers (one thread each) ======================
    // Warp 1 issues the score products, warp 2 the output products: a
    // thread waits ~120 cycles per tcgen05.mma issue whatever its N, so two
    // issuing threads double the rate.  Every product carries its operand
    // terms side by side along N, one MMA per K step.
    // Operand formats: 16-bit K/V use their own format for every operand;
    // FP8 K/V meet E4M3 Q terms and E5M2 P terms.
    constexpr uint32_t f16fmt = DT == LSE_KV_BF16 ? 1u : 0u;
    constexpr uint32_t kvfmt = kF8 ? (kE5 ? 1u : 0u) : f16fmt;
    constexpr uint32_t qfmt = kF8 ? 0u : f16fmt;
    constexpr uint32_t pfmt = kF8 ? 1u : f16fmt;
    const int n_total = (int)(t_stop - t_begin);
    // the whole warp runs the loop (uniform operands); one elected lane issues
    const uint32_t leader = elect_one();
    if (warp == 1) {
      // ---- S^T = K Q^T into the group's score buffer ----
      constexpr uint32_t idesc_qk = instr_desc(kvfmt, qfmt, 0, 0, kTK, kSW);
      TileIter iq;
      iq.init(p, t_begin, t_stop, tab);
      int seg_q = -1;
#pragma unroll 1
      for (int nq = 0; nq < n_total; ++nq, iq.advance(p)) {
        const bool first = iq.seg_start(t_begin), last = iq.seg_end();
        if (first) ++seg_q;
        const int st = nq % NK;
        // the segment's Q, the K tile, and the group's score buffer, which
        // its softmax read out (into registers) at the start of tile nq - 2
        bool go = !first || mbar_wait(bar(kBarQFull + seg_q % QS), (seg_q / QS) & 1, abort_flag,
                                      p.err);
        go = go && mbar_wait(bar(kBarFullK + st), (nq / NK) & 1, abort_flag, p.err);
        go = go && (nq < 2 ||
                    mbar_wait(bar(kBarSEmpty + (nq & 1)), ((nq - 2) >> 1) & 1, abort_flag, p.err));
        if (!__all_sync(0xffffffffu, go)) break;
        tc_fence_after();
        const uint32_t kaddr = k_base + st * Lay::kHalfStage;
        const uint32_t qaddr = q_base + (seg_q % QS) * Lay::kQBytes;
        const uint32_t d = tmem_s(nq & 1);
        // descriptors advance by adding the byte offset / 16 to the start
        // address field
        const uint64_t a0 = smem_desc(kaddr, 16, 1024, kLayoutSw128);
        const uint64_t b0 = smem_desc(qaddr, 16, 1024, kLayoutSw128);
        if constexpr (kF8) {
          // K: one 128-dim region, K steps of 32 bytes
#pragma unroll
          for (int k = 0; k < kD / 32; ++k)
            mma_f8(d, a0 + (uint64_t)(k * 2), b0 + (uint64_t)(k * 2), idesc_qk, k > 0, leader);
        } else {
          // two 64-dim regions of K and of Q; K steps of 32 bytes
#pragma unroll
          for (int k = 0; k < kD / 16; ++k) {
            const uint32_t ka = ((k >> 2) * kRegionBytes + (k & 3) * 32) >> 4;
            const uint32_t kb = ((k >> 2) * 2 * Lay::kQRegion + (k & 3) * 32) >> 4;
            mma_f16(d, a0 + ka, b0 + kb, idesc_qk, k > 0, leader);
          }
        }
        mma_commit(bar(kBarEmptyK + st), leader);
        mma_commit(bar(kBarSFull + (nq & 1)), leader);
        if (last) mma_commit(bar(kBarQEmpty + seg_q % QS), leader);
      }
      // every MMA issued has completed before TMEM is released
      mma_commit(bar(kBarDone), leader);
      mbar_drain(bar(kBarDone), 0);
    } else {
      // ---- O^T += V^T P^T into the piece's output slot ----
      constexpr uint32_t idesc_pv =
          instr_desc(kvfmt, pfmt, 1, 1, kD, (kF8 && !Lay::kPSide) ? kNQ : kN);
      TileIter iv;
      iv.init(p, t_begin, t_stop, tab);
      int seg_v = -1;
#pragma unroll 1
      for (int nv = 0; nv < n_total; ++nv, iv.advance(p)) {
        const bool first = iv.seg_start(t_begin), last = iv.seg_end();
        if (first) ++seg_v;
        const int slot = seg_v % kOS;
        const int st = nv % NV;
        // every group's probabilities of tile nv, its V tile, and (for the
        // piece's first product) the slot's previous piece read out
        bool go = mbar_wait(bar(kBarPFull + nv % PB), (nv / PB) & 1, abort_flag, p.err);
        go = go && mbar_wait(bar(kBarFullV + st), (nv / NV) & 1, abort_flag, p.err);
        if (first)
          go = go && mbar_wait(bar(kBarOEmpty + slot), ((seg_v / kOS) & 1) ^ 1, abort_flag,
                               p.err);
        if (!__all_sync(0xffffffffu, go)) break;
        tc_fence_after();
        const uint32_t vaddr = v_base + st * Lay::kHalfStage;
        const uint32_t d = tmem_o(slot);
        const uint64_t b0 = smem_desc(p_tile(nv), Lay::kPLbo, 128, kLayoutNone);
        if constexpr (kF8) {
          // V^T is MN-major with one 128-byte swizzle atom across the dims
          // (LBO unused); K steps of 32 keys
          const uint64_t a0 = smem_desc(vaddr, 0, 1024, kLayoutSw128);
#pragma unroll
          for (int k = 0; k < kTK / 32; ++k) {
            const uint64_t a = a0 + (uint64_t)(k * 4096 / 16);
            const uint64_t b = b0 + (uint64_t)(k * 4 * Lay::kPLbo / 16);
            if constexpr (Lay::kPSide) {
              // the P terms side by side along N
              mma_f8(d, a, b, idesc_pv, (!first || k > 0) ? 1u : 0u, leader);
            } else {
              // the P terms accumulate into the same columns
#pragma unroll
              for (int t = 0; t < kPTerms; ++t)
                mma_f8(d, a, b + (uint64_t)(t * (kNQ / 16) * 128 / 16), idesc_pv,
                       (!first || k > 0 || t > 0) ? 1u : 0u, leader);
            }
          }
        } else {
          // V^T is MN-major: two 64-dim atoms (LBO), K steps of 16 keys
          const uint64_t a0 = smem_desc(vaddr, kRegionBytes, 1024, kLayoutSw128);
#pragma unroll
          for (int k = 0; k < kTK / 16; ++k)
            mma_f16(d, a0 + (uint64_t)(k * 2048 / 16), b0 + (uint64_t)(k * 2 * Lay::kPLbo / 16),
                    idesc_pv, (!first || k > 0) ? 1u : 0u, leader);
        }
        mma_commit(bar(kBarEmptyV + st), leader);
        mma_commit(bar(kBarPEmpty + nv % PB), leader);
        if (last) mma_commit(bar(kBarOFull + slot), leader);
      }
      mma_commit(bar(kBarDoneV), leader);
      mbar_drain(bar(kBarDoneV), 0);
    }
  } else if (warp == 3) {
    // ============================ Q staging ===============================
    // Every segment after the first, ahead of the score products (softmax
    // group 0 stages the first: it is idle until the first scores arrive,
    // and 128 threads do it faster than one warp).
    // At each segment's start the next segment's Q is prefetched into L2,
    // so its staging (once the slot is free) reads L2, not HBM.
    TileIter it;
    it.init(p, t_begin, t_stop, tab);
    int seg = -1;
    for (; it.valid(); it.advance(p)) {
      if (!it.seg_start(t_begin)) continue;
      const long long nxt = it.seg_first + it.n_tiles;
      if (nxt < t_stop) {
        TileIter nx;
        nx.init(p, nxt, t_stop, tab);
        prefetch_q(p, nx.g, nx.crow0(p), nx.crows(p), lane);
      }
      if (++seg == 0) continue;
      const int slot = seg % QS;
      uint8_t *qs = smem + (q_base - sbase) + slot * Lay::kQBytes;
      const bool okq = stage_q<DT, P8, 32>(
          p, lane, it.g, it.crow0(p), G * it.crows(p), qs, isig_all + slot * 64, [&]() {
            return mbar_wait(bar(kBarQEmpty + slot), ((seg / QS) & 1) ^ 1, abort_flag, p.err);
          });
      if (!okq) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarQFull + slot));
    }
  } else {
    // ============== softmax and epilogue: kG groups of 128 threads ==============
    // Every group works on every tile, each on its share of the (row, head)
    // pairs: group g takes pairs [g H, g H + H), H = P8 / kG, so a tile's
    // softmax is spread over kG groups that never combine results.  Thread j
    // of a group owns key j of the tile (its TMEM lane), reads its share of
    // the key's scores, keeps the key's sums of P per pair
    // in registers over the segment, and the four warps' sums meet once per
    // piece (a warp butterfly, then a fixed-order fold).
    constexpr int kHq = Lay::kH;
    const int grp = (warp - 4) >> 2;
    const int q0 = grp * kHq;                  // this group's first pair
    const int j = tid - 128 - grp * 128;       // key of the tile = TMEM lane (scores)
    const int quarter = warp & 3;              // TMEM lane quarter of this warp
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int bar_id = 1 + grp;
    float *m_run = m_run_all + grp * 64;       // indexed by pair
    float *alpha = alpha_all + grp * 64;       // (at a piece's end: the pairs' row sums)
    float *red = red_all + grp * 4 * 64;       // [warp quarter][pair]
    unsigned long long *masks = masks_all + grp * 64;
    unsigned long long *visk = visk_all + grp * 64;
    float *isg = isig_all + (2 + grp) * 64;    // FP8: the segment's inverse Q scales
    float lacc[kHq];
    TileIter it;
    it.init(p, t_begin, t_stop, tab);
    int n = 0, seg = -1;
    bool had_tile = false, ok = true;
#pragma unroll 1
    for (; it.valid() && ok; it.advance(p), ++n) {
      const bool first = it.seg_start(t_begin), last = it.seg_end();
      const int P = G * it.crows(p);     // (row, head) pairs of the segment
      const int Cctx = it.L - it.R;      // context keys (all rows are drafts)
      const int oslot = (seg + (first ? 1 : 0)) % kOS;
      if (first) {
        ++seg;
        // a finite floor keeps exp2(-inf - m) at 0 (never NaN) for pairs
        // with no visible key yet
        if (j < kHq) m_run[q0 + j] = -FLT_MAX;
#pragma unroll
        for (int q = 0; q < kHq; ++q) lacc[q] = 0.f;
        if (j < it.crows(p)) {
          // the chunk's rows; the default mask is the chain (row r sees drafts
          // 0 .. r of its sequence)
          const int r = it.c * p.rows_per_chunk + j;
          masks[j] = p.row_masks ? p.row_masks[it.row0 + r]
                                 : (r >= 63 ? ~0ull : ((1ull << (r + 1)) - 1ull));
        }
        had_tile = false;
        if (seg == 0 && grp == 0) {
          // the first segment's Q (slot 0, never used before)
          stage_q<DT, P8, 128>(p, j, it.g, it.crow0(p), P, smem + (q_base - sbase), isig_all,
                               [] { return true; });
          named_sync(bar_id, 128);
          if (j == 0) mbar_arrive(bar(kBarQFull));
        }
        bool w = true;
        if constexpr (kF8) {
          // the segment's Q scales: wait for its Q slot, keep a copy, then
          // release the slot (with the score products)
          const int qslot = seg % QS;
          w = mbar_wait(bar(kBarQFull + qslot), (seg / QS) & 1, abort_flag, p.err);
          if (w && j < P8) isg[j] = isig_all[qslot * 64 + j];
        }
        // every thread of the group leaves together when a wait gave up
        if (named_or(bar_id, 128, !w)) {
          ok = false;
          break;
        }
        if (kF8 && j == 0) mbar_arrive(bar(kBarQEmpty + seg % QS));
        if (j < it.R) {
          // draft key j of the sequence: the pairs (G per row) whose row's
          // mask has bit j (read at the next group barrier)
          unsigned long long v = 0;
          const int cr = it.crows(p);
          const unsigned long long row_pairs = G >= 64 ? ~0ull : ((1ull << G) - 1ull);
#pragma unroll 1
          for (int r = 0; r < cr; ++r)
            if ((masks[r] >> j) & 1ull) v |= row_pairs << (r * G);
          visk[j] = v;
        }
        named_sync(bar_id, 128);  // visk and m_run ready for the group
      }
      // ---- tile n: this group's pairs ----
      bool w = mbar_wait(bar(kBarSFull + (n & 1)), (n >> 1) & 1, abort_flag, p.err);
      tc_fence_after();
      // tile record, published by the producer on its own barrier (the K ring
      // may already hold a later tile)
      if (w) w = mbar_wait(bar(kBarInfo + (n & 7)), (n >> 3) & 1, abort_flag, p.err);
      // per-vector scales land with the tile's V (the V slot outlives this
      // pass: its output product waits for this tile's P)
      if (kSc && w) w = mbar_wait(bar(kBarFullV + n % NV), (n / NV) & 1, abort_flag, p.err);
      // (a thread whose wait gave up goes on without side effects up to the
      // group barrier after pass 1, where the whole group learns of it)
      const uint4 inf = w ? tile_info[n & 7] : make_uint4(0u, 0u, 0u, 0u);
      const int key0 = it.tile * kTK;
      const int key = key0 + j;
      const uint32_t both = inf.x & inf.y;
      const bool kvalid = j < (int)inf.z && (both >> (j / box_t) & 1u);
      // Per-vector scales.  The key's score is multiplied by its K scale;
      // its V scale sV enters through the probability: with u = x + log2 sV
      // in place of the score x, the running max and P follow u, P.V sums
      // 2^(u - m) V = 2^(x - m) sV V, and the row sums add 2^(u - m) / sV =
      // 2^(x - m), so the output and log-sum-exp come out unchanged while P
      // stays within the range the unscaled path gives it.  (A V scale
      // below 2^-64 is read as 2^-64; a dead key keeps unit scales.)
      float ks = 1.f, lv = 0.f, ivs = 1.f;
      if constexpr (kSc) {
        if (kvalid) {
          const float *scs = reinterpret_cast<const float *>(
              smem + (sc_base - sbase) + (n % NV) * Lay::kScStage);
          ks = scs[j];
          float vs = scs[kTK + j];
          vs = vs < 0x1p-64f ? 0x1p-64f : vs;  // (NaN stays NaN)
          lv = log2f(vs);
          ivs = 1.f / vs;
        }
      }
      // visibility of this key to each pair, as a bit mask
      unsigned long long vis;
      if (key0 + kTK <= Cctx && inf.z == (uint32_t)kTK && both == full_boxes) {
        vis = ~0ull;  // context tile (pairs past P have zero Q rows; never read)
      } else {
        vis = 0;
        if (kvalid) {
          vis = key < Cctx ? (P >= 64 ? ~0ull : ((1ull << P) - 1ull)) : visk[key - Cctx];
        }
      }
      const uint32_t s_addr = tmem_s(n & 1) + lane_off;
      __syncwarp();
      // pass 1: this group's scores into registers, the score terms summed
      // (16-bit: Q hi and lo blocks; FP8: four Q-term blocks, times the
      // pair's inverse Q scale), -inf where not visible; does any score pass
      // the running max by 2^tau?
      float sv[kHq], mr[kHq];
      // the loads of up to 16 pairs (16-bit) or of 12 or 8 pairs (FP8: four
      // terms each) before one wait
      constexpr int kLd = !kF8 ? (kHq <= 16 ? kHq : 12)
                               : kHq % 12 == 0 ? 12 : kHq % 8 == 0 ? 8 : 4;
#pragma unroll
      for (int i = 0; i < kHq; i += kLd)
        tmem_load_sum<kSW / kNQ, kLd>(s_addr + q0 + i, kNQ, sv + i);
      // the scores are in registers: the next score product into this
      // buffer may overwrite it while the probabilities are built
      tc_fence_before();
      mbar_arrive(bar(kBarSEmpty + (n & 1)));
      if constexpr (kF8) {
#pragma unroll
        for (int i = 0; i < kHq; ++i) sv[i] *= isg[q0 + i];
      }
      if constexpr (kSc) {
#pragma unroll
        for (int i = 0; i < kHq; ++i) sv[i] = fmaf(sv[i], ks, lv);
      }
      if (vis != ~0ull) {
#pragma unroll
        for (int i = 0; i < kHq; ++i)
          if (!((vis >> (q0 + i)) & 1ull)) sv[i] = -INFINITY;
      }
#pragma unroll
      for (int i = 0; i < kHq; i += 4) {
        const float4 m4 = *reinterpret_cast<const float4 *>(m_run + q0 + i);
        mr[i] = m4.x;
        mr[i + 1] = m4.y;
        mr[i + 2] = m4.z;
        mr[i + 3] = m4.w;
      }
      float gap = -INFINITY;
#pragma unroll
      for (int i = 0; i < kHq; ++i) gap = fmaxf(gap, sv[i] - mr[i]);
      // this tile's P buffer is free once the output product that last read
      // it (tile n - PB) has completed
      if (n >= PB && w)
        w = mbar_wait(bar(kBarPEmpty + n % PB), ((n / PB) - 1) & 1, abort_flag, p.err);
      // one group barrier per tile in the common case: does any thread need
      // the rescale, or has any wait given up?
      if (named_or(bar_id, 128, !w || gap > kTau)) {
        if (named_or(bar_id, 128, !w)) {  // (uniform over the group)
          ok = false;
          break;
        }
        // per-pair maximum over the tile's keys: each warp folds its 32
        // keys by a butterfly, and the four warps' maxima meet in red
#pragma unroll
        for (int i = 0; i < kHq; i += 4) {
          const float wm = warp_reduce4<true>(sv + i, lane);
          if ((lane & 7) == 0) red[quarter * 64 + q0 + i + ((lane >> 3) & 3)] = wm;
        }
        named_sync(bar_id, 128);
        if (j < kHq) {
          const int q = q0 + j;
          const float mo = m_run[q];
          const float mn = fmaxf(mo, fmaxf(fmaxf(red[q], red[64 + q]),
                                           fmaxf(red[128 + q], red[192 + q])));
          alpha[q] = ex2(mo - mn);
          m_run[q] = mn;
        }
        named_sync(bar_id, 128);
#pragma unroll
        for (int i = 0; i < kHq; i += 4) {
          const float4 m4 = *reinterpret_cast<const float4 *>(m_run + q0 + i);
          mr[i] = m4.x;
          mr[i + 1] = m4.y;
          mr[i + 2] = m4.z;
          mr[i + 3] = m4.w;
        }
#pragma unroll
        for (int i = 0; i < kHq; ++i) lacc[i] *= alpha[q0 + i];
        if (had_tile) {
          // rescale this group's output columns once every earlier output
          // product has completed (they complete in issue order: the one of
          // tile n - 1 covers them all)
          const bool wo = mbar_wait(bar(kBarPEmpty + (n - 1) % PB), ((n - 1) / PB) & 1,
                                    abort_flag, p.err);
          if (named_or(bar_id, 128, !wo)) {
            ok = false;
            break;
          }
          tc_fence_after();
          __syncwarp();
          const uint32_t ob = tmem_o(oslot) + lane_off;
#pragma unroll 1
          for (int blk = 0; blk < kN / Lay::kOBlk; ++blk)
#pragma unroll 1
            for (int i = 0; i < kHq; i += 4) {
              const uint32_t col = (uint32_t)(blk * Lay::kOBlk + q0 + i);
              float v[4];
              tmem_load_sum4<1>(ob + col, 0, v);
#pragma unroll
              for (int u = 0; u < 4; ++u) v[u] *= alpha[q0 + i + u];
              tmem_st4(ob + col, v);
            }
          tmem_st_wait();
        }
      }
      // pass 2: probabilities of this group's pairs -> the tile's P tile, row
      // j (16-bit: hi block then lo block; FP8: P 2^7 as kPTerms E5M2 terms,
      // a block each), and this thread's sums of them per pair
      uint8_t *prow = smem + (p_tile(n) - sbase) + (j >> 3) * Lay::kPLbo + (j & 7) * 16;
#pragma unroll
      for (int i = 0; i < kHq; i += 4) {
        float e[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) e[u] = ex2(sv[i + u] - mr[i + u]);  // 0 where not visible
        if constexpr (kF8) {
#pragma unroll
          for (int u = 0; u < 4; ++u) e[u] *= (float)(1 << kPScaleLog2);
          uint32_t wt[kPTerms];
          e5_terms4<kPTerms>(e, wt);
          // 16 FP8 columns per core matrix: term t's pair q sits in column
          // t kNQ + q
#pragma unroll
          for (int t = 0; t < kPTerms; ++t) {
            const int col = t * kNQ + q0 + i;
            *reinterpret_cast<uint32_t *>(prow + (col >> 4) * 128 + (col & 15)) = wt[t];
          }
        } else {
          uint32_t h0, l0, h1, l1;
          split2<DT>(e[0], e[1], h0, l0);
          split2<DT>(e[2], e[3], h1, l1);
          // 8 16-bit columns per core matrix: pair q's hi term in column q,
          // its lo term in column P8 + q
          const int ch = q0 + i, cl = P8 + q0 + i;
          *reinterpret_cast<uint2 *>(prow + (ch >> 3) * 128 + (ch & 7) * 2) = make_uint2(h0, h1);
          *reinterpret_cast<uint2 *>(prow + (cl >> 3) * 128 + (cl & 7) * 2) = make_uint2(l0, l1);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) lacc[i + u] = kSc ? fmaf(e[u], ivs, lacc[i + u])
                                                      : lacc[i + u] + e[u];
      }
      if (!kvalid && grp == 0) {
        // a dead slot may hold any bits: give it a zero V row (P is 0 there)
        mbar_wait(bar(kBarFullV + n % NV), (n / NV) & 1, abort_flag, p.err);
        uint8_t *v0 = smem + (v_base - sbase) + (n % NV) * Lay::kHalfStage + j * 128;
        constexpr int kChunks = kF8 ? 8 : 16;  // 16-byte chunks of the row
#pragma unroll 1
        for (int c = 0; c < kChunks; ++c)
          *reinterpret_cast<uint4 *>(v0 + (c >> 3) * kRegionBytes + (c & 7) * 16) =
              make_uint4(0, 0, 0, 0);
      }
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(bar(kBarPFull + n % PB));
      had_tile = true;

      if (last) {
        // ---- epilogue of the piece: this group's pairs ----
        const bool we = mbar_wait(bar(kBarOFull + oslot), (seg / kOS) & 1, abort_flag, p.err);
        if (named_or(bar_id, 128, !we)) {
          ok = false;
          break;
        }
        // the row sums of P: each warp folds its 32 keys per pair, the four
        // warps' sums are added in a fixed order (results repeat bit for bit)
#pragma unroll
        for (int i = 0; i < kHq; i += 4) {
          const float ws = warp_reduce4<false>(lacc + i, lane);
          if ((lane & 7) == 0) red[quarter * 64 + q0 + i + ((lane >> 3) & 3)] = ws;
        }
        named_sync(bar_id, 128);
        if (j < kHq) {
          const int q = q0 + j;
          alpha[q] = ((red[q] + red[64 + q]) + red[128 + q]) + red[192 + q];
        }
        named_sync(bar_id, 128);
        tc_fence_after();
        __syncwarp();
        // the piece: its place among the segment's pieces
        const long long pos0 = it.seg_first + (long long)W * (it.seg_id + 1);
        const int c_first = cta_of_pos(pos0, UW, C);
        const int c_last = cta_of_pos(pos0 + it.n_tiles - 1, UW, C);
        const int n_pieces = c_last - c_first + 1, piece = cta - c_first;
        const bool direct = tp.fused && n_pieces == 1;  // the final output, no partial
        const int d = j;  // output lane = head dim
        const uint32_t ob = tmem_o(oslot) + lane_off;
        const long long row_stride = (long long)p.n_q_heads * tp.n_slots * kD;
        const long long base =
            ((long long)it.crow0(p) * p.n_q_heads + it.g * G) * tp.n_slots + piece;
#pragma unroll 1
        for (int i = 0; i < kHq; i += 4) {
          float o[4];
          // the output blocks (hi and lo, or the P terms) summed
          tmem_load_sum4<kN / Lay::kOBlk>(ob + q0 + i, Lay::kOBlk, o);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int q = q0 + i + u;
            if (q < P) {
              const float lt = alpha[q];
              const float v = lt > 0.f ? o[u] * rcp(lt) : 0.f;
              // log2-sum-exp (FP8 sums carry P's factor 2^7)
              const float lse2 =
                  lt > 0.f ? m_run[q] + lg2(lt) - (kF8 ? kPScaleLog2 : 0) : -INFINITY;
              const int r = pair_row[q];
              const int h = it.g * G + (q - r * G);
              if (direct) {
                const long long oi = (long long)(it.crow0(p) + r) * p.n_q_heads + h;
                p.out[oi * kD + d] = v;
                if (d == q && p.lse_out) p.lse_out[oi] = lse2 * 0.69314718055994530942f;
              } else {
                const long long idx =
                    base + r * row_stride / kD + (long long)(q - r * G) * tp.n_slots;
                p.o_part[idx * kD + d] = v;
                if (d == q) p.lse_part[idx] = lse2;
              }
            }
          }
        }
        // every thread of the group has read the pairs' maxima and sums
        // before any thread resets them at its next segment
        tc_fence_before();
        if (tp.fused && n_pieces > 1) __threadfence();
        named_sync(bar_id, 128);
        mbar_arrive(bar(kBarOEmpty + oslot));
        if (tp.fused && n_pieces > 1) {
          // this group's share of the piece's partial is written (and fenced
          // above): count it on the segment (kG arrivals per piece); the CTA
          // merges its share of the segment once every piece is in (end phase)
          if (j == 0) {
            atomicAdd(p.seg_count + 2 * it.seg_id, 1u);
            if (grp == 0) {
              const int k = *n_end;
              if (k < 2) {
                end_rec[k] = EndRec{it.seg_id, n_pieces, piece, it.crow0(p), it.crows(p), it.g};
                *n_end = k + 1;
              }
            }
          }
        }
      }
    }
  }

  // ---- teardown --------------------------------------------------------------
  tc_fence_before();
  __syncthreads();
  // (the K/V ring is idle: the end phase's scratch)
  if (tp.fused)
    fused_end_merge<kThreads / 32, kG>(tp, end_rec, *n_end, abort_flag, had_all,
                    reinterpret_cast<float *>(smem + (k_base - sbase)));
  // TMEM is released last: only its owner fences after the barrier (the
  // fence there held the merge back by several microseconds)
  if (warp == 1) {
    tc_fence_after();
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(Lay::kTmemCols)
                 : "memory");
  }
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

template <int DT, int P8, bool kSc>
int launch_tc(const TcParams &tp, int smem, cudaStream_t st) {
  auto k = partial_tcgen05_kernel<DT, P8, kSc>;
  static lse_detail::SmemAllowed allowed;  // per device ordinal
  const int e = lse_detail::allow_dynamic_smem(k, smem, allowed);
  if (e) return e;
  if (!tp.fused) {
    k<<<tp.n_ctas, tc_threads<P8>(), smem, st>>>(tp);
    return (int)cudaGetLastError();
  }
  // the fused merge waits (bounded) for other CTAs' pieces: a cooperative
  // launch, so every CTA of the grid is resident at once (or the launch fails)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tp.n_ctas);
  cfg.blockDim = dim3(tc_threads<P8>());
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return (int)cudaLaunchKernelEx(&cfg, k, tp);
}

template <int DT, bool kSc>
int launch_tc_p(const TcParams &tp, int p8, int smem, cudaStream_t st) {
  switch (p8) {
    case 8: return launch_tc<DT, 8, kSc>(tp, smem, st);
    case 16: return launch_tc<DT, 16, kSc>(tp, smem, st);
    case 24: return launch_tc<DT, 24, kSc>(tp, smem, st);
    case 32: return launch_tc<DT, 32, kSc>(tp, smem, st);
    case 48: return launch_tc<DT, 48, kSc>(tp, smem, st);
  }
  return (int)cudaErrorInvalidValue;
}

template <int DT>
int smem_for_p(int p8, int k_stages, int v_stages, int q_slots, int p_bufs, bool scaled) {
  switch (p8) {
    case 8: return TcLayout<DT, 8>::smem_bytes(k_stages, v_stages, q_slots, p_bufs, scaled);
    case 16: return TcLayout<DT, 16>::smem_bytes(k_stages, v_stages, q_slots, p_bufs, scaled);
    case 24: return TcLayout<DT, 24>::smem_bytes(k_stages, v_stages, q_slots, p_bufs, scaled);
    case 32: return TcLayout<DT, 32>::smem_bytes(k_stages, v_stages, q_slots, p_bufs, scaled);
    case 48: return TcLayout<DT, 48>::smem_bytes(k_stages, v_stages, q_slots, p_bufs, scaled);
  }
  return -1;
}

int smem_for(int dtype, int p8, int k_stages, int v_stages, int q_slots, int p_bufs,
             bool scaled) {
  // the two 16-bit formats share a layout, and so do the two 8-bit ones
  return is_f8(dtype)
             ? smem_for_p<LSE_KV_FP8_E4M3>(p8, k_stages, v_stages, q_slots, p_bufs, scaled)
             : smem_for_p<LSE_KV_BF16>(p8, k_stages, v_stages, q_slots, p_bufs, scaled);
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

// Shared-memory configuration: the most K and V tile slots, then a second P
// tile (the next tile's probabilities are written while the output product
// reads this one) and a second Q slot (overlapping Q staging with the end of
// the previous segment) when they fit as well.  The slots are split about
// 1 : 2 between the K and the V ring (at least two each, K at most
// kMaxStages, V at most 8): a K slot is free again once its score product is
// done, a V slot only after the softmax of its tile and its output product.
int lse_tc_smem(int dtype, int p8, int scaled, int smem_optin, int *k_stages, int *v_stages,
                int *q_slots, int *p_bufs) {
  if (scaled && !is_f8(dtype)) return -1;
  for (int slots = kMaxStages + 8; slots >= 4; --slots) {
    const int nk = slots / 3 < 2 ? 2 : (slots / 3 > kMaxStages ? kMaxStages : slots / 3);
    const int nv = slots - nk;
    if (nv < 2 || nv > 8) continue;
    for (int pb = 2; pb >= 1; --pb)
      for (int qs = 2; qs >= 1; --qs) {
        const int b = smem_for(dtype, p8, nk, nv, qs, pb, scaled != 0);
        if (b > 0 && b <= smem_optin) {
          *k_stages = nk;
          *v_stages = nv;
          *q_slots = qs;
          *p_bufs = pb;
          return b;
        }
      }
  }
  return -1;
}

int lse_tc_key_tile() { return kTK; }

int lse_tc_build_maps(const uint64_t *chunk_base, int n_chunks, size_t chunk_bytes,
                      int n_kv_heads, int dtype, int box_tokens, void *maps_out) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = get_encode();
  if (!enc) return (int)cudaErrorNotSupported;
  if (n_chunks > LSE_MAX_TMA_CHUNKS) return (int)cudaErrorInvalidValue;
  CUtensorMap *maps = static_cast<CUtensorMap *>(maps_out);
  // a chunk as [tokens][rows][128 bytes]: 16-bit K/V give two 64-dim rows
  // per kv head, FP8 one 128-dim row.  The bytes are described to the TMA
  // unit as 8-byte elements (16 per row) whatever the storage format: the
  // 128-byte swizzle moves 16-byte pieces, so shared memory receives the same
  // layout, and the copy engine handles far fewer elements per byte.
  const bool f8 = is_f8(dtype);
  const int esize = f8 ? 1 : 2;
  const int rows_per_head = f8 ? 1 : 2;
  const uint64_t row = (uint64_t)n_kv_heads * kD * esize;  // bytes per token, all kv heads
  for (int c = 0; c < n_chunks; ++c) {
    cuuint64_t dims[3] = {16, (cuuint64_t)n_kv_heads * rows_per_head,
                          (cuuint64_t)(chunk_bytes / row)};
    cuuint64_t strides[2] = {128, row};
    cuuint32_t box[3] = {16, 1, (cuuint32_t)box_tokens};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(&maps[c], CU_TENSOR_MAP_DATA_TYPE_UINT64, 3,
                     reinterpret_cast<void *>(chunk_base[c]), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     // L2 fills no wider than one kv head's row (128 bytes
                     // for FP8, 256 for 16-bit), so no fill drags in a
                     // neighbouring head's bytes
                     f8 ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B : CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return (int)cudaErrorInvalidValue;
  }
  return 0;
}

size_t lse_tc_map_bytes() { return sizeof(CUtensorMap); }

int lse_launch_partial_tcgen05(const LseKernelParams &p, const void *maps, int n_maps,
                               int dtype, int p8, int scaled, int n_ctas, int n_slots,
                               int k_stages, int v_stages, int q_slots, int p_bufs,
                               int box_tokens, int smem, int fused, int withhold_tile,
                               void *stream) {
  static_assert(sizeof(TcParams) < 30000, "kernel parameter block too large");
  TcParams tp;
  memset(&tp, 0, sizeof tp);
  memcpy(tp.maps, maps, sizeof(CUtensorMap) * n_maps);
  tp.p = p;
  tp.n_ctas = n_ctas;
  tp.n_slots = n_slots;
  tp.k_stages = k_stages;
  tp.v_stages = v_stages;
  tp.q_slots = q_slots;
  tp.p_bufs = p_bufs;
  tp.box_tokens = box_tokens;
  tp.fused = fused;
  tp.withhold_tile = withhold_tile;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  switch (dtype) {
    case LSE_KV_BF16:
      return scaled ? (int)cudaErrorInvalidValue : launch_tc_p<LSE_KV_BF16, false>(tp, p8, smem, st);
    case LSE_KV_F16:
      return scaled ? (int)cudaErrorInvalidValue : launch_tc_p<LSE_KV_F16, false>(tp, p8, smem, st);
    case LSE_KV_FP8_E4M3:
      return scaled ? launch_tc_p<LSE_KV_FP8_E4M3, true>(tp, p8, smem, st)
                    : launch_tc_p<LSE_KV_FP8_E4M3, false>(tp, p8, smem, st);
    case LSE_KV_FP8_E5M2:
      return scaled ? launch_tc_p<LSE_KV_FP8_E5M2, true>(tp, p8, smem, st)
                    : launch_tc_p<LSE_KV_FP8_E5M2, false>(tp, p8, smem, st);
  }
  return (int)cudaErrorInvalidValue;
}
