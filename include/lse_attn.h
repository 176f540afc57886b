/*
 * lse_attn.h — split-KV paged attention for single-token decode and
 * speculative verification over a fragment-addressed K/V cache, on NVIDIA
 * B200 (sm_100a).
 *
 * What is computed (sources: the LSE README (Geramy/LSE), "KV cache
 * formats"; LSE releases, v0.4.19 "Long-context split attention", v0.4.20
 * "K/V memory management and automatic split attention", v0.4.21 "joint
 * decode attention", v0.4.14 "Improvements"):
 *
 *   For sequence s with L_s keys, the last R_s of which are the query rows
 *   (context C_s = L_s - R_s), query row r (position C_s + r), query head h,
 *   kv head g = h / (Hq / Hkv):
 *     visible(j)  <=>  j < C_s  or  bit (j - C_s) of mask_r is set
 *     x_j  = softmax_scale * <q[r][h], K[j][g]>
 *     out  = sum_vis exp(x_j - m) V[j][g] / sum_vis exp(x_j - m),  m = max_vis x_j
 *     lse  = m + ln sum_vis exp(x_j - m)
 *   mask_r defaults to the chain (rows 0..r); for a draft tree it is the row
 *   itself plus its ancestors (nodes in topological order, R_s <= 64).
 *
 *   K/V elements are stored as FP32, FP16, BF16, FP8-E4M3 ("fp8") or
 *   FP8-E5M2 ("bf8"); accumulation, softmax state and output are FP32.
 *   The work is split along the keys into partitions whose count comes from
 *   page-table capacity and on-chip memory limits (lse_attn_plan); each
 *   partition writes a normalised partial output and its log-sum-exp
 *   (lse_attn_run); a merge pass combines them (lse_attn_merge).  A
 *   partition with no live key loads nothing and writes nothing.
 *
 * Memory layout
 *   Arena: n_chunks device allocations ("arenas" on the pages) of chunk_bytes
 *   each, cut into fragments of fragment_bytes.  Fragment id f lives in chunk
 *   f / (chunk_bytes / fragment_bytes) at byte offset
 *   (f % (chunk_bytes / fragment_bytes)) * fragment_bytes.  A fragment holds
 *   T = fragment_bytes / (Hkv * D * esize) consecutive tokens of K (or of V)
 *   for every kv head, token-major: [token][kv_head][dim].  K and V use
 *   separate fragments and separate page tables.
 *   Page tables: int32 [n_seqs][max_pages_per_seq]; key j of sequence s is
 *   token j % T of fragment table[s][j / T].  Entries past the live pages are
 *   ignored.
 *   q:   FP32 [total_rows][Hq][D]; the rows of sequence s are
 *        row_offsets[s] .. row_offsets[s+1]-1.
 *   out: FP32 [total_rows][Hq][D];  lse_out (optional): FP32 [total_rows][Hq].
 *
 * Ownership and threading
 *   The library never allocates, frees or owns device memory: the caller
 *   allocates the arena chunks, page tables, q, out and the workspace (size
 *   from lse_attn_plan).  Handles (arena, plan) are host objects owned by the
 *   library and released by their destroy calls.  Device pointers are passed
 *   as plain pointers; every launch goes to the caller's cudaStream_t (passed
 *   as void*; NULL = legacy default stream).  No call synchronises except
 *   the read-error calls.  Several host threads may run and merge with one
 *   plan at the same time (each with its own workspace); a call that
 *   changes an arena (alloc, free, add_chunk, set_scales) must not overlap a
 *   call that reads it (planning, run, merge, append).
 *
 * Errors
 *   Every call returns LSE_OK (0) or an lse_status code.  When err is not
 *   NULL and a call fails, *err receives a message the caller releases with
 *   lse_free (the convention of libLSE's C API in the LSE README).  Host
 *   checks cover every size and shape.  Device-resident inputs (page tables,
 *   lengths, masks) are not read on the host by lse_attn_run; the kernels
 *   bound-check them instead: a bad fragment id or length sets a bit in the
 *   workspace's error word (read with lse_attn_read_error), the offending
 *   keys are treated as absent, and no out-of-bounds access is made.
 *   lse_attn_validate checks host copies of those arrays up front.
 */
#ifndef LSE_ATTN_H
#define LSE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LSE_API __attribute__((visibility("default")))
#else
#define LSE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LSE_OK = 0,
  LSE_ERR_INVALID_ARG = 1,      /* a size, shape, pointer or dtype is out of range */
  LSE_ERR_UNSUPPORTED = 2,      /* valid, but no kernel here handles it             */
  LSE_ERR_OUT_OF_FRAGMENTS = 3, /* the arena has fewer free fragments than asked   */
  LSE_ERR_CUDA = 4,             /* a CUDA runtime call or launch failed             */
  LSE_ERR_NO_MEMORY = 5,        /* a host allocation failed                         */
  LSE_ERR_BAD_INPUT = 6         /* validated input violates the layout/mask rules   */
} lse_status;

typedef enum {
  LSE_KV_F32 = 0,
  LSE_KV_F16 = 1,
  LSE_KV_BF16 = 2,
  LSE_KV_FP8_E4M3 = 3, /* OCP E4M3: finite only, max 448, NaN = S.1111.111 */
  LSE_KV_FP8_E5M2 = 4  /* OCP E5M2: IEEE-style inf and NaN                  */
} lse_kv_dtype;

/* Bits of the device error word (lse_attn_read_error). */
#define LSE_DEVERR_BAD_FRAGMENT 0x1u /* a page-table entry named no fragment   */
#define LSE_DEVERR_TIMEOUT 0x4u      /* a pipeline wait ran out (~2 s); the call aborted */
#define LSE_DEVERR_BAD_LENGTH 0x2u   /* L_s > capacity, R_s > L_s, R_s > max rows or rows past max_total_rows */

#define LSE_MAX_CHUNKS 64     /* arena chunks a kernel can address          */
#define LSE_MAX_TMA_CHUNKS 64 /* chunks the tensor-core kernel can address (every chunk
                                 an arena can have: one TMA descriptor per chunk) */
#define LSE_MAX_ROWS_PER_SEQ 64    /* rows per sequence of the verify kernels (64-bit masks) */
#define LSE_MAX_BLOCK_ROWS 32768   /* rows per sequence of a long query block (chain only) */

typedef struct lse_kv_arena lse_kv_arena;
typedef struct lse_attn_plan_s lse_attn_plan_t;

/* ---------------------------------------------------------------------------
 * K/V arena (LSE releases, v0.4.20: 256 MiB arenas of 256 KiB fragments,
 * shared across layers and sessions; free slots are reused before another
 * arena is added; growth never moves existing fragments).
 * ------------------------------------------------------------------------- */

/* Describe an arena over caller-owned device chunks.
 *   chunk_bases: n_chunks device pointers (host array), each 256-byte aligned
 *                and chunk_bytes long; 1 <= n_chunks <= LSE_MAX_CHUNKS.
 *   fragment_bytes must divide chunk_bytes, be a multiple of
 *   Hkv * D * esize and of 16.  head_dim in {64, 128, 256}.
 *   All fragments start free.  *out receives the handle. */
LSE_API int lse_kv_arena_create(void *const *chunk_bases, int n_chunks, size_t chunk_bytes,
                        size_t fragment_bytes, int kv_dtype, int n_kv_heads, int head_dim,
                        lse_kv_arena **out, char **err);

/* Append one more caller-owned chunk (growth without copying).  Its
 * fragments get the next ids; *first_id (optional) receives the first. */
LSE_API int lse_kv_arena_add_chunk(lse_kv_arena *arena, void *chunk_base, int32_t *first_id,
                           char **err);

/* Take n free fragment ids, lowest id first (so earlier chunks fill before
 * later ones); on LSE_ERR_OUT_OF_FRAGMENTS nothing is taken. */
LSE_API int lse_kv_arena_alloc(lse_kv_arena *arena, int n, int32_t *frag_ids_out, char **err);

/* Return fragment ids; a double free or an unknown id is LSE_ERR_INVALID_ARG
 * and frees nothing. */
LSE_API int lse_kv_arena_free(lse_kv_arena *arena, int n, const int32_t *frag_ids, char **err);

typedef struct {
  int32_t tokens_per_fragment; /* T */
  int32_t n_fragments;         /* all chunks */
  int32_t n_free;
  int32_t n_chunks;
  int32_t n_empty_chunks;      /* chunks whose fragments are all free (releasable) */
} lse_kv_arena_info;

LSE_API int lse_kv_arena_query(const lse_kv_arena *arena, lse_kv_arena_info *info);

/* Per-vector FP32 scales of an 8-bit arena (LSE README, "KV cache formats":
 * fp8 and bf8 "with scales", 33,280 bytes per token where the elements take
 * 32,768: one FP32 scale per (token, kv head) of K and of V).  A stored
 * vector times its scale is the key or value: K[j][g][:] =
 * decode(stored K[j][g][:]) * sK[j][g], and V likewise.
 *   scales: device FP32 array, 16-byte aligned, caller-owned, paged like
 *           the vectors: fragment id f owns the block of T * Hkv floats at
 *           scales + f * Hkv * T, laid out [kv_head][token], so K scales sit
 *           in the blocks of K fragments and V scales in those of V
 *           fragments.  n_floats >= n_fragments * Hkv * T (a chunk added
 *           later needs a larger array, set again).  Scales are finite and
 *           non-negative; a V scale below 2^-64 may be read as 2^-64 (the
 *           value it weights changes by less than 2^-64 of the output).
 *   scales = NULL removes them (unit scales).
 * Attention reads the scales; lse_kv_append writes the scales of the
 * vectors it stores.  Plans record whether the arena had scales when they
 * were made; running a plan after the arena's scales were added or removed
 * is LSE_ERR_INVALID_ARG.
 * Errors: LSE_ERR_UNSUPPORTED for 16-bit or FP32 arenas, LSE_ERR_INVALID_ARG
 * for a misaligned or short array. */
LSE_API int lse_kv_arena_set_scales(lse_kv_arena *arena, float *scales, int64_t n_floats,
                                    char **err);

LSE_API void lse_kv_arena_destroy(lse_kv_arena *arena);

/* ---------------------------------------------------------------------------
 * Plan (LSE releases, v0.4.20: the partition count is derived from the
 * actual K/V table capacity and checked against on-chip memory limits;
 * partitions past a sequence's live keys are skipped).
 *   n_seqs, max_rows_per_seq (<= 64), max_total_rows (>= rows of one call),
 *   n_q_heads (multiple of Hkv), max_pages_per_seq (page-table row length:
 *   the capacity).  Uses the current CUDA device's SM count and shared
 *   memory limit.  *workspace_bytes receives the device workspace size the
 *   caller allocates (256-byte aligned; zero it once with
 *   lse_attn_workspace_init).  The plan does not depend on live lengths, so
 *   one plan serves every step up to the capacity.
 * ------------------------------------------------------------------------- */
LSE_API int lse_attn_plan(const lse_kv_arena *arena, int n_seqs, int max_rows_per_seq,
                  int max_total_rows, int n_q_heads, int max_pages_per_seq,
                  lse_attn_plan_t **out, size_t *workspace_bytes, char **err);

/* Device figures the planner uses.  lse_attn_plan reads them from the
 * current CUDA device; lse_attn_plan_ex takes them from the caller and then
 * makes no CUDA call (planning for another device, or on a host without
 * one).  ctas_per_sm = 0 asks the CUDA occupancy calculator. */
typedef struct {
  int32_t n_sms;          /* streaming multiprocessors                     */
  int32_t smem_optin;     /* shared memory per block, opt-in maximum       */
  int32_t ctas_per_sm;    /* resident partial-pass CTAs per SM (0 = query)  */
  int32_t allow_tcgen05;  /* 1: the tensor-core kernel may be chosen        */
} lse_device_limits;

LSE_API int lse_attn_plan_ex(const lse_kv_arena *arena, int n_seqs, int max_rows_per_seq,
                             int max_total_rows, int n_q_heads, int max_pages_per_seq,
                             const lse_device_limits *limits, lse_attn_plan_t **out,
                             size_t *workspace_bytes, char **err);

/* Kernel families a plan can select. */
#define LSE_KERNEL_CUDA_CORE 0 /* FP32 math on CUDA cores (any dtype, any P) */
#define LSE_KERNEL_TCGEN05 1   /* tensor-core (tcgen05) partial pass           */
#define LSE_KERNEL_PREFILL 2   /* tensor-core pass for long query blocks (rows as M) */

/* For LSE_KERNEL_CUDA_CORE the partitions are fixed ranges of K_p keys,
 * n_splits = ceil(capacity / K_p), and partitions past a sequence's live
 * keys are skipped.  For LSE_KERNEL_TCGEN05 the partial pass is persistent
 * (one CTA per SM): the live 128-key tiles of all (sequence, kv head) pairs
 * are laid end to end and cut into equal contiguous ranges, one per CTA;
 * a CTA's share of one (sequence, kv head) is a piece, which yields one
 * partial (the CTA combines its two softmax warpgroups), so n_splits =
 * min(CTAs, capacity tiles) bounds the partials of one (sequence, kv head);
 * keys_per_split reports the tile (128); capacity without live keys is
 * never visited. */
typedef struct {
  int32_t n_splits;        /* partial slots per (row, head)                  */
  int32_t keys_per_split;  /* K_p (CUDA-core) or the key tile (tcgen05)      */
  int32_t kernel;          /* LSE_KERNEL_*                                  */
  int32_t key_tile;        /* keys per pipeline stage                      */
  int32_t pairs;           /* (row, head) pairs per kv head: G * max rows   */
  int32_t smem_bytes;      /* dynamic shared memory of the partial kernel  */
  int32_t ctas;            /* partial-pass CTAs when persistent, else 0     */
  int64_t workspace_bytes;
  int32_t stages;          /* tensor-core kernels: K ring depth (long query
                              blocks: K/V ring depth), else 0              */
  int32_t q_slots;         /* tensor-core kernel: Q ring depth, else 0        */
  int32_t p_bufs;          /* tensor-core kernel: P tiles per softmax group   */
  int32_t rows_per_chunk;  /* tensor-core kernel: query rows per segment (a
                              sequence with more rows is split into row
                              chunks, each reading its keys), else 0       */
  int32_t scaled;          /* 1: made for an arena with per-vector scales  */
  int32_t v_stages;        /* verify tensor-core kernel: V ring depth, else 0 */
  int32_t merge_in_pass;   /* 1: lse_attn_forward merges inside the partial
                              pass's launch (tensor-core plans); 0: a
                              partial launch and a merge launch            */
} lse_attn_plan_info;

LSE_API int lse_attn_plan_query(const lse_attn_plan_t *plan, lse_attn_plan_info *info);

/* Same partition rule as lse_attn_plan, for explicit device figures (no
 * CUDA call): capacity_keys = max_pages * T; units = n_seqs * Hkv;
 * slots = n_sms * ctas_per_sm; key_tile = the kernel's keys per stage.
 * K_p = clamp(roundup(ceil(capacity_keys * units / slots), key_tile),
 *             key_tile, roundup(capacity_keys, key_tile));
 * n_splits = ceil(capacity_keys / K_p).  Returns n_splits; *keys_per_split
 * receives K_p. */
LSE_API int lse_attn_split_rule(int64_t capacity_keys, int units, int n_sms, int ctas_per_sm,
                        int key_tile, int32_t *keys_per_split);

/* Zero the workspace's error word and the fused pass's segment counters
 * (once after allocation; any time to clear). */
LSE_API int lse_attn_workspace_init(const lse_attn_plan_t *plan, void *workspace, void *stream,
                            char **err);

LSE_API void lse_attn_plan_destroy(lse_attn_plan_t *plan);

/* ---------------------------------------------------------------------------
 * Partial pass (LSE releases, v0.4.19: one partial family, verifier rows
 * share K/V loads; v0.4.21: K/V reads shared across query heads and rows).
 *   q:           device FP32 [total_rows][Hq][D]
 *   k_pages,
 *   v_pages:     device int32 [n_seqs][max_pages_per_seq]
 *   seq_lens:    device int32 [n_seqs]      (L_s, query rows included)
 *   row_offsets: device int32 [n_seqs + 1]  (R_s = difference, <= max rows)
 *   row_masks:   device uint64 [total_rows] ancestor masks, or NULL = chain
 *   softmax_scale: multiplies <q, k> (1/sqrt(D) in the usual case)
 *   workspace:   device, workspace_bytes, 256-byte aligned
 *   stream:      cudaStream_t
 * Each live partition of each (sequence, kv head) reads its K/V tiles once
 * for every query head of the group and every query row.
 * ------------------------------------------------------------------------- */
LSE_API int lse_attn_run(const lse_attn_plan_t *plan, const float *q, const int32_t *k_pages,
                 const int32_t *v_pages, const int32_t *seq_lens, const int32_t *row_offsets,
                 const uint64_t *row_masks, float softmax_scale, void *workspace, void *stream,
                 char **err);

/* ---------------------------------------------------------------------------
 * Merge pass (LSE releases, v0.4.19: one merge family).  For each row and
 * head, with partials (o_p, lse_p) over the live partitions:
 *   M = max_p lse_p, w_p = exp(lse_p - M),
 *   out = sum_p w_p o_p / sum_p w_p,  lse = M + ln sum_p w_p.
 *   out: device FP32 [total_rows][Hq][D]; lse_out: device FP32
 *   [total_rows][Hq] or NULL.  seq_lens / row_offsets as given to run.
 * ------------------------------------------------------------------------- */
LSE_API int lse_attn_merge(const lse_attn_plan_t *plan, const int32_t *seq_lens,
                   const int32_t *row_offsets, const void *workspace, float *out,
                   float *lse_out, void *stream, char **err);

/* ---------------------------------------------------------------------------
 * Partial and merge passes in one call (LSE releases, v0.4.19: one partial
 * and one merge family; v0.4.20: empty partitions skipped).  Arguments as
 * lse_attn_run plus lse_attn_merge's out / lse_out; the result equals
 * lse_attn_run followed by lse_attn_merge up to FP32 rounding.
 * For tensor-core plans the merge runs inside the partial pass's launch: a
 * CTA whose share of a (sequence, kv head) is the whole of it writes the
 * final output directly; the partials of a shared one are merged at the end
 * of the launch by the CTAs that computed them, after a bounded wait for
 * the other pieces.  That launch is cooperative (every CTA resident at
 * once; the call fails with LSE_ERR_CUDA where the device cannot hold the
 * grid) and uses the workspace's segment counters, which each call leaves
 * at zero.  After a call that set a device error bit, read it with
 * lse_attn_read_error (which then also clears the counters) or call
 * lse_attn_workspace_init before the next call.  For CUDA-core plans this
 * is lse_attn_run then lse_attn_merge.
 * ------------------------------------------------------------------------- */
LSE_API int lse_attn_forward(const lse_attn_plan_t *plan, const float *q, const int32_t *k_pages,
                             const int32_t *v_pages, const int32_t *seq_lens,
                             const int32_t *row_offsets, const uint64_t *row_masks,
                             float softmax_scale, void *workspace, float *out, float *lse_out,
                             void *stream, char **err);

/* ---------------------------------------------------------------------------
 * Host-side validation of HOST copies of the device inputs: every live page
 * names a fragment of the arena (sequences may share read-only fragments),
 * L_s <= capacity,
 * 1 <= R_s <= min(L_s, 64) (R_s = 0 allowed: the sequence is idle), total
 * rows <= max_total_rows, each mask has bit r set and no bit above r.
 * Returns LSE_OK or LSE_ERR_BAD_INPUT with a message naming the first fault.
 * ------------------------------------------------------------------------- */
LSE_API int lse_attn_validate(const lse_attn_plan_t *plan, const int32_t *k_pages,
                      const int32_t *v_pages, const int32_t *seq_lens,
                      const int32_t *row_offsets, const uint64_t *row_masks, char **err);

/* Read (and clear) the workspace's device error word.  Synchronises the
 * stream.  *device_error receives LSE_DEVERR_* bits, 0 when clean; when it
 * is not, the fused pass's segment counters are cleared as well. */
LSE_API int lse_attn_read_error(const lse_attn_plan_t *plan, void *workspace, void *stream,
                        uint32_t *device_error, char **err);

/* ---------------------------------------------------------------------------
 * K/V append (LSE releases, v0.4.20 "K/V memory management and automatic
 * split attention": K/V tensors live in fragments reached through each
 * sequence's page tables; a decode or verify step writes its new tokens'
 * K/V there before attending).  Writes the K and V vectors of new tokens into
 * their fragments, cast from FP32 to the arena's storage format: the nearest
 * value of the format, ties to even; F16 and BF16 overflow to infinity,
 * E4M3 and E5M2 saturate at their largest finite value (448, 57344).
 * When the arena has per-vector scales (lse_kv_arena_set_scales), each
 * vector's scale is its largest magnitude over the format's largest finite
 * value (1 for an all-zero vector), written to its entry of the scale
 * array, and each element is stored as the FP32 quotient element / scale,
 * rounded as above.
 *
 * Token i of sequence s, new_offsets[s] <= i < new_offsets[s+1], goes to key
 * position seq_lens_before[s] + i - new_offsets[s] of s (page = position / T,
 * slot = position % T, T the fragment's tokens), the same element layout the
 * attention passes read ([token][kv_head][dim] inside a fragment).
 *   k_new, v_new      device, FP32 [total_new][n_kv_heads][head_dim]
 *   k_pages, v_pages  device, int32 [n_seqs][max_pages]; the pages holding
 *                     the new positions must already name fragments
 *   seq_lens_before   device, int32 [n_seqs]: keys stored before this append
 *   new_offsets       device, int32 [n_seqs + 1], ascending, new_offsets[0] = 0
 *   total_new         host: new_offsets[n_seqs] (sizes the launch)
 *   err_word          device uint32, or NULL: LSE_DEVERR_BAD_FRAGMENT is ORed
 *                     in when a position is past its page table or a page
 *                     names no fragment (that vector is not written),
 *                     LSE_DEVERR_BAD_LENGTH when a token belongs to no
 *                     sequence (new_offsets not ascending)
 * Head dims 64, 128 and 256.  Asynchronous on `stream`; allocates nothing;
 * the caller owns every buffer.  Returns LSE_OK, LSE_ERR_INVALID_ARG (NULL
 * or out-of-range arguments), LSE_ERR_UNSUPPORTED (head dim) or
 * LSE_ERR_CUDA (launch failure).
 * ------------------------------------------------------------------------- */
LSE_API int lse_kv_append(const lse_kv_arena *arena, int n_seqs, int max_pages,
                          const float *k_new, const float *v_new, const int32_t *k_pages,
                          const int32_t *v_pages, const int32_t *seq_lens_before,
                          const int32_t *new_offsets, int total_new, uint32_t *err_word,
                          void *stream, char **err);

/* ---------------------------------------------------------------------------
 * No-allocation variant (the pages have no counterpart: it exists for
 * callers that cannot allocate device memory when attention runs, such as
 * plugin or custom-op hosts that hand a kernel only its inputs and outputs,
 * and serving loops whose device memory is fixed at start-up, so that no
 * allocation may happen after warm-up).
 * Runs lse_attn_run then lse_attn_merge on `stream` with the workspace taken
 * from a static device array of LSE_STATIC_SCRATCH_BYTES that the library
 * holds on every GPU that loads it until the process exits.  Arguments as
 * lse_attn_run and lse_attn_merge (device pointers; out [total_rows][Hq][D],
 * lse_out optional).  It calls no cudaMalloc, cudaFree or other allocating
 * routine.
 *   - A plan whose workspace_bytes exceed LSE_STATIC_SCRATCH_BYTES is
 *     rejected with LSE_ERR_UNSUPPORTED and a message.
 *   - The first call on each device looks the array's device address up
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.
 *   - Every call shares the one array and leaves its contents behind; the
 *     device error word is cleared at the start of each call.  Calls whose
 *     GPU work overlaps (other streams, other threads) race on the array:
 *     serialise them.
 *   - The device error word of the latest call (bad fragment id, bad
 *     length, pipeline timeout) is read with lse_attn_static_read_error.
 * ------------------------------------------------------------------------- */
#define LSE_STATIC_SCRATCH_BYTES (32u << 20)

LSE_API int lse_attn_forward_static(const lse_attn_plan_t *plan, const float *q,
                                    const int32_t *k_pages, const int32_t *v_pages,
                                    const int32_t *seq_lens, const int32_t *row_offsets,
                                    const uint64_t *row_masks, float softmax_scale, float *out,
                                    float *lse_out, void *stream, char **err);

/* Read (and clear) the device error word of the static scratch on the
 * current device: the LSE_DEVERR_* bits the latest lse_attn_forward_static
 * call on this device left (0 when clean).  Synchronises the stream.  Like
 * the static call itself it allocates nothing; the first use on a device
 * looks the scratch address up.  No counterpart on the pages. */
LSE_API int lse_attn_static_read_error(void *stream, uint32_t *device_error, char **err);

/* Testing the bounded waits (no counterpart on the pages).  Every wait of
 * the tensor-core pass gives up after about 2 s, sets LSE_DEVERR_TIMEOUT,
 * drains the copies and products in flight, releases TMEM and returns, so
 * a fault upstream never leaves the GPU blocked.  After this call every
 * later launch of `plan` skips loading each CTA's tile of local index
 * `tile` (nothing arrives on that tile's barriers), so those waits run out;
 * tile = -1 restores normal loading.  For tests only.  Returns
 * LSE_ERR_UNSUPPORTED for plans of other kernels. */
LSE_API int lse_attn_test_withhold_tile(lse_attn_plan_t *plan, int tile);

/* Release a string returned through an err argument. */
LSE_API void lse_free(void *p);

/* Static description of a status code. */
LSE_API const char *lse_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* LSE_ATTN_H */
