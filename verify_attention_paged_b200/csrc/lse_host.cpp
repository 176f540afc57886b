// Host side of liblse_attn.so: the K/V arena's fragment bookkeeping, the
// split planner, input validation and the C-ABI entry points that launch
// the kernels.  See include/lse_attn.h for the contract of every call.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "lse_internal.h"

namespace {

int fail(char **err, int status, const char *fmt, ...) {
  if (err) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    size_t n = strlen(buf) + 1;
    char *m = static_cast<char *>(malloc(n));
    if (m) memcpy(m, buf, n);
    *err = m;
  }
  return status;
}

int cuda_fail(char **err, int code, const char *what) {
  return fail(err, LSE_ERR_CUDA, "%s: %s", what, lse_cuda_error_string(code));
}

int elem_size(int dtype) {
  switch (dtype) {
    case LSE_KV_F32: return 4;
    case LSE_KV_F16:
    case LSE_KV_BF16: return 2;
    case LSE_KV_FP8_E4M3:
    case LSE_KV_FP8_E5M2: return 1;
  }
  return 0;
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

extern "C" {

const char *lse_status_string(int status) {
  switch (status) {
    case LSE_OK: return "ok";
    case LSE_ERR_INVALID_ARG: return "invalid argument";
    case LSE_ERR_UNSUPPORTED: return "unsupported";
    case LSE_ERR_OUT_OF_FRAGMENTS: return "out of fragments";
    case LSE_ERR_CUDA: return "CUDA error";
    case LSE_ERR_NO_MEMORY: return "out of host memory";
    case LSE_ERR_BAD_INPUT: return "bad input";
  }
  return "unknown status";
}

void lse_free(void *p) { free(p); }

// ---- arena -----------------------------------------------------------------

int lse_kv_arena_create(void *const *chunk_bases, int n_chunks, size_t chunk_bytes,
                        size_t fragment_bytes, int kv_dtype, int n_kv_heads, int head_dim,
                        lse_kv_arena **out, char **err) {
  if (!out) return fail(err, LSE_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  const int es = elem_size(kv_dtype);
  if (!es) return fail(err, LSE_ERR_INVALID_ARG, "unknown kv dtype %d", kv_dtype);
  if (head_dim != 64 && head_dim != 128 && head_dim != 256)
    return fail(err, LSE_ERR_INVALID_ARG, "head_dim %d not in {64, 128, 256}", head_dim);
  if (n_kv_heads <= 0) return fail(err, LSE_ERR_INVALID_ARG, "n_kv_heads %d", n_kv_heads);
  if (n_chunks < 1 || n_chunks > LSE_MAX_CHUNKS || !chunk_bases)
    return fail(err, LSE_ERR_INVALID_ARG, "n_chunks %d not in [1, %d]", n_chunks,
                LSE_MAX_CHUNKS);
  const size_t row = size_t(n_kv_heads) * head_dim * es;
  if (fragment_bytes == 0 || fragment_bytes % row || fragment_bytes % 16)
    return fail(err, LSE_ERR_INVALID_ARG,
                "fragment_bytes %zu must be a positive multiple of 16 and of Hkv*D*esize = %zu",
                fragment_bytes, row);
  if (chunk_bytes == 0 || chunk_bytes % fragment_bytes)
    return fail(err, LSE_ERR_INVALID_ARG, "chunk_bytes %zu is not a multiple of %zu",
                chunk_bytes, fragment_bytes);
  const size_t fpc = chunk_bytes / fragment_bytes;
  if (fpc * size_t(LSE_MAX_CHUNKS) > size_t(INT32_MAX) || fragment_bytes / row > (1u << 30))
    return fail(err, LSE_ERR_INVALID_ARG, "too many fragments");
  for (int c = 0; c < n_chunks; ++c) {
    if (!chunk_bases[c] || (reinterpret_cast<uintptr_t>(chunk_bases[c]) & 255u))
      return fail(err, LSE_ERR_INVALID_ARG, "chunk %d base is NULL or not 256-byte aligned", c);
  }
  lse_kv_arena *a = new (std::nothrow) lse_kv_arena;
  if (!a) return fail(err, LSE_ERR_NO_MEMORY, "arena");
  a->chunk_bytes = chunk_bytes;
  a->fragment_bytes = fragment_bytes;
  a->dtype = kv_dtype;
  a->n_kv_heads = n_kv_heads;
  a->head_dim = head_dim;
  a->esize = es;
  a->tokens_per_fragment = int(fragment_bytes / row);
  a->frags_per_chunk = int(fpc);
  for (int c = 0; c < n_chunks; ++c)
    a->chunk_base.push_back(reinterpret_cast<uint64_t>(chunk_bases[c]));
  a->used.assign(fpc * n_chunks, 0);
  a->chunk_live.assign(n_chunks, 0);
  a->n_free = int32_t(fpc * n_chunks);
  *out = a;
  return LSE_OK;
}

int lse_kv_arena_add_chunk(lse_kv_arena *a, void *chunk_base, int32_t *first_id, char **err) {
  if (!a) return fail(err, LSE_ERR_INVALID_ARG, "arena is NULL");
  if (int(a->chunk_base.size()) >= LSE_MAX_CHUNKS)
    return fail(err, LSE_ERR_UNSUPPORTED, "arena already has %d chunks", LSE_MAX_CHUNKS);
  if (!chunk_base || (reinterpret_cast<uintptr_t>(chunk_base) & 255u))
    return fail(err, LSE_ERR_INVALID_ARG, "chunk base is NULL or not 256-byte aligned");
  const int32_t first = int32_t(a->used.size());
  a->chunk_base.push_back(reinterpret_cast<uint64_t>(chunk_base));
  a->used.resize(a->used.size() + a->frags_per_chunk, 0);
  a->chunk_live.push_back(0);
  a->n_free += a->frags_per_chunk;
  if (first_id) *first_id = first;
  return LSE_OK;
}

int lse_kv_arena_set_scales(lse_kv_arena *a, float *scales, int64_t n_floats, char **err) {
  if (!a) return fail(err, LSE_ERR_INVALID_ARG, "arena is NULL");
  if (!scales) {
    a->scales = nullptr;
    a->n_scales = 0;
    return LSE_OK;
  }
  if (a->dtype != LSE_KV_FP8_E4M3 && a->dtype != LSE_KV_FP8_E5M2)
    return fail(err, LSE_ERR_UNSUPPORTED, "per-vector scales go with the 8-bit formats");
  if (reinterpret_cast<uintptr_t>(scales) & 15u)
    return fail(err, LSE_ERR_INVALID_ARG, "scale array is not 16-byte aligned");
  const int64_t need = int64_t(a->used.size()) * a->n_kv_heads * a->tokens_per_fragment;
  if (n_floats < need)
    return fail(err, LSE_ERR_INVALID_ARG, "scale array holds %lld floats; the arena's %d "
                "fragments need %lld", (long long)n_floats, int(a->used.size()),
                (long long)need);
  a->scales = scales;
  a->n_scales = n_floats;
  return LSE_OK;
}

int lse_kv_arena_alloc(lse_kv_arena *a, int n, int32_t *ids, char **err) {
  if (!a || n < 0 || (n > 0 && !ids)) return fail(err, LSE_ERR_INVALID_ARG, "bad arguments");
  if (n > a->n_free)
    return fail(err, LSE_ERR_OUT_OF_FRAGMENTS, "asked for %d fragments, %d free", n, a->n_free);
  int32_t f = a->scan_from;
  const int32_t total = int32_t(a->used.size());
  for (int i = 0; i < n; ++i) {
    while (f < total && a->used[f]) ++f;
    a->used[f] = 1;
    a->chunk_live[f / a->frags_per_chunk]++;
    ids[i] = f++;
  }
  a->n_free -= n;
  a->scan_from = f;
  return LSE_OK;
}

int lse_kv_arena_free(lse_kv_arena *a, int n, const int32_t *ids, char **err) {
  if (!a || n < 0 || (n > 0 && !ids)) return fail(err, LSE_ERR_INVALID_ARG, "bad arguments");
  const int32_t total = int32_t(a->used.size());
  // check everything first so that a bad list frees nothing
  std::vector<int32_t> sorted(ids, ids + n);
  std::sort(sorted.begin(), sorted.end());
  for (int i = 0; i < n; ++i) {
    const int32_t f = sorted[i];
    if (f < 0 || f >= total) return fail(err, LSE_ERR_INVALID_ARG, "fragment %d unknown", f);
    if (!a->used[f]) return fail(err, LSE_ERR_INVALID_ARG, "fragment %d is not in use", f);
    if (i && sorted[i - 1] == f) return fail(err, LSE_ERR_INVALID_ARG, "fragment %d twice", f);
  }
  for (int i = 0; i < n; ++i) {
    const int32_t f = ids[i];
    a->used[f] = 0;
    a->chunk_live[f / a->frags_per_chunk]--;
    if (f < a->scan_from) a->scan_from = f;
  }
  a->n_free += n;
  return LSE_OK;
}

int lse_kv_arena_query(const lse_kv_arena *a, lse_kv_arena_info *info) {
  if (!a || !info) return LSE_ERR_INVALID_ARG;
  info->tokens_per_fragment = a->tokens_per_fragment;
  info->n_fragments = int32_t(a->used.size());
  info->n_free = a->n_free;
  info->n_chunks = int32_t(a->chunk_base.size());
  info->n_empty_chunks = 0;
  for (int32_t live : a->chunk_live) info->n_empty_chunks += live == 0;
  return LSE_OK;
}

void lse_kv_arena_destroy(lse_kv_arena *a) { delete a; }

// ---- planner -------------------------------------------------------------------

int lse_attn_split_rule(int64_t capacity_keys, int units, int n_sms, int ctas_per_sm,
                        int key_tile, int32_t *keys_per_split) {
  if (capacity_keys <= 0 || units <= 0 || n_sms <= 0 || ctas_per_sm <= 0 || key_tile <= 0)
    return 0;
  const int64_t slots = int64_t(n_sms) * ctas_per_sm;
  int64_t kp = round_up(ceil_div(capacity_keys * units, slots), key_tile);
  kp = std::max<int64_t>(kp, key_tile);
  kp = std::min<int64_t>(kp, round_up(capacity_keys, key_tile));
  if (keys_per_split) *keys_per_split = int32_t(kp);
  return int(ceil_div(capacity_keys, kp));
}

int lse_attn_plan(const lse_kv_arena *a, int n_seqs, int max_rows, int max_total_rows,
                  int n_q_heads, int max_pages, lse_attn_plan_t **out, size_t *ws_bytes,
                  char **err) {
  return lse_attn_plan_ex(a, n_seqs, max_rows, max_total_rows, n_q_heads, max_pages, nullptr,
                          out, ws_bytes, err);
}

int lse_attn_plan_ex(const lse_kv_arena *a, int n_seqs, int max_rows, int max_total_rows,
                     int n_q_heads, int max_pages, const lse_device_limits *limits,
                     lse_attn_plan_t **out, size_t *ws_bytes, char **err) {
  if (!out) return fail(err, LSE_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (!a) return fail(err, LSE_ERR_INVALID_ARG, "arena is NULL");
  if (n_seqs < 1) return fail(err, LSE_ERR_INVALID_ARG, "n_seqs %d", n_seqs);
  if (max_rows < 1 || max_rows > LSE_MAX_BLOCK_ROWS)
    return fail(err, LSE_ERR_INVALID_ARG, "max_rows_per_seq %d not in [1, %d]", max_rows,
                LSE_MAX_BLOCK_ROWS);
  if (max_total_rows < 1 || max_total_rows > n_seqs * max_rows)
    return fail(err, LSE_ERR_INVALID_ARG, "max_total_rows %d not in [1, %d]", max_total_rows,
                n_seqs * max_rows);
  if (n_q_heads < a->n_kv_heads || n_q_heads % a->n_kv_heads)
    return fail(err, LSE_ERR_INVALID_ARG, "n_q_heads %d is not a multiple of n_kv_heads %d",
                n_q_heads, a->n_kv_heads);
  if (max_pages < 1) return fail(err, LSE_ERR_INVALID_ARG, "max_pages_per_seq %d", max_pages);
  const int64_t cap_keys = int64_t(max_pages) * a->tokens_per_fragment;
  if (cap_keys > INT32_MAX / 2)
    return fail(err, LSE_ERR_INVALID_ARG, "capacity of %lld keys too large",
                (long long)cap_keys);
  if (int64_t(n_seqs) * max_rows > (1 << 24) || int64_t(n_q_heads) > 4096)
    return fail(err, LSE_ERR_INVALID_ARG, "too many rows or heads");

  int n_sms = 0, smem_optin = 0, ctas_given = 0, allow_tc = 1, ce = 0;
  if (limits) {
    n_sms = limits->n_sms;
    smem_optin = limits->smem_optin;
    ctas_given = limits->ctas_per_sm;
    allow_tc = limits->allow_tcgen05;
    if (n_sms < 1 || smem_optin < 1 || ctas_given < 0)
      return fail(err, LSE_ERR_INVALID_ARG, "bad device limits");
  } else {
    int dev = 0;
    ce = (int)cudaGetDevice(&dev);
    if (ce) return cuda_fail(err, ce, "cudaGetDevice");
    ce = (int)cudaDeviceGetAttribute(&n_sms, cudaDevAttrMultiProcessorCount, dev);
    if (ce) return cuda_fail(err, ce, "cudaDeviceGetAttribute(SM count)");
    ce = (int)cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (ce) return cuda_fail(err, ce, "cudaDeviceGetAttribute(shared memory)");
    int major = 0;
    ce = (int)cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (ce) return cuda_fail(err, ce, "cudaDeviceGetAttribute(compute capability)");
    allow_tc = major == 10;  // tcgen05 needs sm_100
  }

  lse_attn_plan_t *pl = new (std::nothrow) lse_attn_plan_t;
  if (!pl) return fail(err, LSE_ERR_NO_MEMORY, "plan");
  pl->arena = a;
  pl->n_seqs = n_seqs;
  pl->max_rows = max_rows;
  pl->max_total_rows = max_total_rows;
  pl->n_q_heads = n_q_heads;
  pl->n_kv_heads = a->n_kv_heads;
  pl->group = n_q_heads / a->n_kv_heads;
  pl->head_dim = a->head_dim;
  pl->dtype = a->dtype;
  pl->max_pages = max_pages;
  pl->tokens_per_fragment = a->tokens_per_fragment;
  pl->pairs = pl->group * max_rows;
  pl->n_sms = n_sms;
  pl->scaled = a->scales != nullptr;

  // kernel choice and its on-chip memory check.  The tensor-core kernel
  // takes 16-bit and FP8 K/V with head_dim 128 and fragments whose token
  // count tiles evenly into 128-key tiles.  A kv head's (row, head) pairs
  // must fit one score tile (48); more rows are cut into row chunks of
  // floor(48 / G) rows, each reading the sequence's keys again.
  const int T = a->tokens_per_fragment;
  const bool t_ok = (T % 128 == 0) || (T >= 8 && T % 8 == 0 && 128 % T == 0);
  const int max_tile_pairs = 48;
  const int rows_per_chunk =
      pl->pairs <= max_tile_pairs ? max_rows : max_tile_pairs / pl->group;
  const int p8 = rows_per_chunk > 0 ? lse_tc_pairs_bucket(pl->group * rows_per_chunk) : -1;
  int tc_stages = 0, tc_v_stages = 0, tc_q_slots = 0, tc_p_bufs = 0;
  const int tc_smem =
      p8 > 0 ? lse_tc_smem(a->dtype, p8, pl->scaled, smem_optin, &tc_stages, &tc_v_stages,
                           &tc_q_slots, &tc_p_bufs)
             : -1;
  if (max_rows > LSE_MAX_ROWS_PER_SEQ) {
    // a long query block (chain rows only): the rows-as-M tensor-core pass
    const int rt = lse_pf_row_tile();
    const int64_t row_tiles = int64_t(n_seqs) * ceil_div(max_rows, rt);
    const char *why = !allow_tc ? "a device with tcgen05"
                      : a->dtype == LSE_KV_F32 ? "16-bit or FP8 K/V"
                      : a->head_dim != 128 ? "head_dim 128"
                      : !t_ok ? "fragments of a multiple or divisor of 128 tokens (>= 8)"
                      : pl->scaled ? "an arena without per-vector scales"
                      : row_tiles > lse_pf_max_row_tiles() ? "at most 256 row tiles of 128 rows"
                      : nullptr;
    int pf_stages = 0;
    const int pf_smem = why ? -1 : lse_pf_smem(a->dtype, smem_optin, &pf_stages);
    if (!why && pf_smem < 0) why = "more shared memory";
    if (why) {
      delete pl;
      return fail(err, LSE_ERR_UNSUPPORTED, "more than %d rows per sequence (a long query "
                  "block) needs %s", LSE_MAX_ROWS_PER_SEQ, why);
    }
    pl->kernel = LSE_KERNEL_PREFILL;
    pl->key_tile = lse_tc_key_tile();
    pl->smem_bytes = pf_smem;
    pl->stages = pf_stages;
    pl->box_tokens = T < pl->key_tile ? T : pl->key_tile;
    pl->ctas = n_sms;
    pl->rows_per_chunk = rt;
    // two partial slots of a 128-row tile per CTA: its first and last
    // segments, the only ones it may share with other CTAs
    pl->n_splits = 2;
    pl->keys_per_split = pl->key_tile;
    pl->n_seg_max = int(row_tiles) * n_q_heads;
  } else if (allow_tc && a->dtype != LSE_KV_F32 && a->head_dim == 128 &&
      t_ok && p8 > 0 && tc_smem > 0) {
    const int tile = lse_tc_key_tile();
    pl->kernel = LSE_KERNEL_TCGEN05;
    pl->key_tile = tile;
    pl->smem_bytes = tc_smem;
    pl->stages = tc_stages;
    pl->v_stages = tc_v_stages;
    pl->q_slots = tc_q_slots;
    pl->p_bufs = tc_p_bufs;
    pl->pairs_bucket = p8;
    pl->rows_per_chunk = rows_per_chunk;
    pl->box_tokens = T < tile ? T : tile;
    pl->ctas = n_sms;
    const int64_t cap_tiles = ceil_div(cap_keys, tile);
    // a segment (sequence, row chunk, kv head) has at most min(CTAs, tiles)
    // pieces, one partial each (the CTA combines its two softmax groups)
    pl->n_splits = int(std::min<int64_t>(n_sms, cap_tiles));
    pl->keys_per_split = tile;
    pl->n_seg_max = n_seqs * int(ceil_div(max_rows, rows_per_chunk)) * a->n_kv_heads;
  } else {
    pl->kernel = LSE_KERNEL_CUDA_CORE;
    pl->key_tile = 32;
    pl->smem_bytes = lse_partial_cuda_core_smem(a->head_dim);
    if (pl->smem_bytes < 0 || pl->smem_bytes > smem_optin) {
      delete pl;
      return fail(err, LSE_ERR_UNSUPPORTED, "partial kernel needs %d bytes of shared memory, "
                  "device allows %d", pl->smem_bytes, smem_optin);
    }
    int ctas_per_sm = ctas_given;
    if (ctas_per_sm == 0) {
      ce = lse_partial_cuda_core_occupancy(a->dtype, a->head_dim, pl->smem_bytes, &ctas_per_sm);
      if (ce) {
        delete pl;
        return cuda_fail(err, ce, "occupancy query");
      }
    }
    ctas_per_sm = std::max(1, ctas_per_sm);
    int32_t kp = 0;
    pl->n_splits = lse_attn_split_rule(cap_keys, n_seqs * a->n_kv_heads, n_sms, ctas_per_sm,
                                       pl->key_tile, &kp);
    pl->keys_per_split = kp;
  }

  const size_t n_part = pl->kernel == LSE_KERNEL_PREFILL
                            ? size_t(n_sms) * 2 * lse_pf_row_tile()
                            : size_t(max_total_rows) * n_q_heads * pl->n_splits;
  pl->ws_cnt_off = kWsHeader;
  pl->ws_o_off = align256(pl->ws_cnt_off + size_t(pl->n_seg_max) * 2 * sizeof(uint32_t));
  pl->ws_lse_off = align256(pl->ws_o_off + n_part * a->head_dim * sizeof(float));
  pl->ws_bytes = align256(pl->ws_lse_off + n_part * sizeof(float));
  if (ws_bytes) *ws_bytes = pl->ws_bytes;
  *out = pl;
  return LSE_OK;
}

int lse_attn_plan_query(const lse_attn_plan_t *pl, lse_attn_plan_info *info) {
  if (!pl || !info) return LSE_ERR_INVALID_ARG;
  info->n_splits = pl->n_splits;
  info->keys_per_split = pl->keys_per_split;
  info->kernel = pl->kernel;
  info->key_tile = pl->key_tile;
  info->pairs = pl->pairs;
  info->smem_bytes = pl->smem_bytes;
  info->ctas = pl->kernel != LSE_KERNEL_CUDA_CORE ? pl->ctas : 0;
  info->workspace_bytes = int64_t(pl->ws_bytes);
  const bool tc = pl->kernel == LSE_KERNEL_TCGEN05, pf = pl->kernel == LSE_KERNEL_PREFILL;
  info->stages = tc || pf ? pl->stages : 0;
  info->q_slots = tc ? pl->q_slots : 0;
  info->p_bufs = tc ? pl->p_bufs : 0;
  info->rows_per_chunk = tc || pf ? pl->rows_per_chunk : 0;
  info->scaled = pl->scaled;
  info->v_stages = tc ? pl->v_stages : 0;
  info->merge_in_pass = pl->kernel != LSE_KERNEL_CUDA_CORE ? 1 : 0;
  return LSE_OK;
}

void lse_attn_plan_destroy(lse_attn_plan_t *pl) { delete pl; }

int lse_attn_test_withhold_tile(lse_attn_plan_t *pl, int tile) {
  if (!pl || tile < -1) return LSE_ERR_INVALID_ARG;
  if (pl->kernel != LSE_KERNEL_TCGEN05) return LSE_ERR_UNSUPPORTED;
  pl->withhold_tile = tile;
  return LSE_OK;
}

int lse_attn_workspace_init(const lse_attn_plan_t *pl, void *ws, void *stream, char **err) {
  if (!pl || !ws) return fail(err, LSE_ERR_INVALID_ARG, "plan or workspace is NULL");
  // the error word and the fused merge's segment counters
  int ce = (int)cudaMemsetAsync(ws, 0, pl->ws_o_off, reinterpret_cast<cudaStream_t>(stream));
  if (ce) return cuda_fail(err, ce, "cudaMemsetAsync");
  return LSE_OK;
}

// ---- run / merge ----------------------------------------------------------------

static int fill_params(const lse_attn_plan_t *pl, void *ws, LseKernelParams &p, char **err) {
  const lse_kv_arena *a = pl->arena;
  if (reinterpret_cast<uintptr_t>(ws) & 255u)
    return fail(err, LSE_ERR_INVALID_ARG, "workspace is not 256-byte aligned");
  if (pl->scaled != (a->scales != nullptr))
    return fail(err, LSE_ERR_INVALID_ARG, pl->scaled ? "plan made with per-vector scales, "
                "arena has none now" : "arena has per-vector scales; the plan was made "
                "without them");
  if (a->scales &&
      a->n_scales < int64_t(a->used.size()) * a->n_kv_heads * a->tokens_per_fragment)
    return fail(err, LSE_ERR_INVALID_ARG, "the arena grew past its scale array");
  memset(&p, 0, sizeof p);
  p.scales = a->scales;
  for (size_t c = 0; c < a->chunk_base.size(); ++c) p.chunk_base[c] = a->chunk_base[c];
  p.fragment_bytes = (long long)a->fragment_bytes;
  p.frags_per_chunk = a->frags_per_chunk;
  p.n_fragments = int(a->used.size());
  p.n_q_heads = pl->n_q_heads;
  p.n_kv_heads = pl->n_kv_heads;
  p.group = pl->group;
  p.head_dim = pl->head_dim;
  p.tokens_per_fragment = pl->tokens_per_fragment;
  p.max_pages = pl->max_pages;
  p.n_splits = pl->n_splits;
  p.keys_per_split = pl->keys_per_split;
  p.max_rows = pl->max_rows;
  p.max_total_rows = pl->max_total_rows;
  p.n_seqs = pl->n_seqs;
  p.rows_per_chunk = pl->rows_per_chunk > 0 ? pl->rows_per_chunk : 1;
  char *base = static_cast<char *>(ws);
  p.err = reinterpret_cast<unsigned int *>(base);
  p.seg_count = reinterpret_cast<unsigned int *>(base + pl->ws_cnt_off);
  p.o_part = reinterpret_cast<float *>(base + pl->ws_o_off);
  p.lse_part = reinterpret_cast<float *>(base + pl->ws_lse_off);
  return LSE_OK;
}

int lse_kv_append(const lse_kv_arena *a, int n_seqs, int max_pages, const float *k_new,
                  const float *v_new, const int32_t *k_pages, const int32_t *v_pages,
                  const int32_t *seq_lens_before, const int32_t *new_offsets, int total_new,
                  uint32_t *err_word, void *stream, char **err) {
  if (!a) return fail(err, LSE_ERR_INVALID_ARG, "arena is NULL");
  if (n_seqs < 1 || max_pages < 1 || total_new < 0)
    return fail(err, LSE_ERR_INVALID_ARG, "n_seqs %d, max_pages %d, total_new %d", n_seqs,
                max_pages, total_new);
  if (a->head_dim != 64 && a->head_dim != 128 && a->head_dim != 256)
    return fail(err, LSE_ERR_UNSUPPORTED, "head_dim %d (append takes 64, 128, 256)",
                a->head_dim);
  if (!k_pages || !v_pages || !seq_lens_before || !new_offsets ||
      (total_new > 0 && (!k_new || !v_new)))
    return fail(err, LSE_ERR_INVALID_ARG, "a required device pointer is NULL");
  if (int64_t(n_seqs) * max_pages > INT32_MAX || int64_t(total_new) * a->n_kv_heads > INT32_MAX)
    return fail(err, LSE_ERR_INVALID_ARG, "too many pages or tokens");
  if (total_new == 0) return LSE_OK;
  AppendParams p;
  memset(&p, 0, sizeof p);
  for (size_t c = 0; c < a->chunk_base.size(); ++c) p.chunk_base[c] = a->chunk_base[c];
  p.fragment_bytes = (long long)a->fragment_bytes;
  p.frags_per_chunk = a->frags_per_chunk;
  p.n_fragments = int(a->used.size());
  p.tokens_per_fragment = a->tokens_per_fragment;
  p.n_kv_heads = a->n_kv_heads;
  p.n_seqs = n_seqs;
  p.max_pages = max_pages;
  p.total_new = total_new;
  p.k_new = k_new;
  p.v_new = v_new;
  p.k_pages = k_pages;
  p.v_pages = v_pages;
  p.seq_lens_before = seq_lens_before;
  p.new_offsets = new_offsets;
  p.err = err_word;
  if (a->scales) {
    if (a->n_scales < int64_t(a->used.size()) * a->n_kv_heads * a->tokens_per_fragment)
      return fail(err, LSE_ERR_INVALID_ARG, "the arena grew past its scale array");
    p.scales = a->scales;
  }
  const int ce = lse_launch_kv_append(p, a->dtype, a->head_dim, stream);
  if (ce) return cuda_fail(err, ce, "append kernel launch");
  return LSE_OK;
}

// The partial pass; with `fused` (tensor-core plans only) the same launch
// also merges and writes out / lse_out.
static int launch_partial(const lse_attn_plan_t *pl, const float *q, const int32_t *k_pages,
                          const int32_t *v_pages, const int32_t *seq_lens,
                          const int32_t *row_offsets, const uint64_t *row_masks,
                          float softmax_scale, void *ws, float *out, float *lse_out, int fused,
                          void *stream, char **err) {
  if (!pl) return fail(err, LSE_ERR_INVALID_ARG, "plan is NULL");
  if (!q || !k_pages || !v_pages || !seq_lens || !row_offsets || !ws)
    return fail(err, LSE_ERR_INVALID_ARG, "a required device pointer is NULL");
  if (!std::isfinite(softmax_scale))
    return fail(err, LSE_ERR_INVALID_ARG, "softmax_scale is not finite");
  LseKernelParams p;
  int st = fill_params(pl, ws, p, err);
  if (st) return st;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.q = q;
  p.k_pages = k_pages;
  p.v_pages = v_pages;
  p.seq_lens = seq_lens;
  p.row_offsets = row_offsets;
  p.row_masks = reinterpret_cast<const unsigned long long *>(row_masks);
  p.out = out;
  p.lse_out = lse_out;
  int ce = 0;
  if (pl->kernel == LSE_KERNEL_PREFILL && !fused)
    return fail(err, LSE_ERR_UNSUPPORTED, "a long-query-block plan (more than %d rows per "
                "sequence) runs through lse_attn_forward", LSE_MAX_ROWS_PER_SEQ);
  if (pl->kernel == LSE_KERNEL_PREFILL && row_masks)
    return fail(err, LSE_ERR_INVALID_ARG, "row masks take at most %d rows per sequence; a "
                "long query block is a chain (row_masks = NULL)", LSE_MAX_ROWS_PER_SEQ);
  if (pl->kernel != LSE_KERNEL_CUDA_CORE) {
    const lse_kv_arena *a = pl->arena;
    const int nch = int(a->chunk_base.size());
    if (nch > LSE_MAX_TMA_CHUNKS)  // (the arena itself holds at most this many)
      return fail(err, LSE_ERR_UNSUPPORTED, "arena has %d chunks; the tensor-core kernel "
                  "addresses at most %d", nch, LSE_MAX_TMA_CHUNKS);
    std::lock_guard<std::mutex> lock(pl->maps_mutex);
    if (pl->maps_chunks != nch) {
      pl->maps.assign(lse_tc_map_bytes() * nch, 0);
      ce = lse_tc_build_maps(a->chunk_base.data(), nch, a->chunk_bytes, a->n_kv_heads,
                             a->dtype, pl->box_tokens, pl->maps.data());
      if (ce) {
        pl->maps_chunks = 0;
        return cuda_fail(err, ce, "building TMA descriptors");
      }
      pl->maps_chunks = nch;
    }
    if (pl->kernel == LSE_KERNEL_PREFILL)
      ce = lse_launch_prefill_tcgen05(p, pl->maps.data(), nch, pl->dtype, pl->ctas, pl->stages,
                                      pl->box_tokens, pl->smem_bytes, stream);
    else
      ce = lse_launch_partial_tcgen05(p, pl->maps.data(), nch, pl->dtype, pl->pairs_bucket,
                                      pl->scaled, pl->ctas, pl->n_splits, pl->stages,
                                      pl->v_stages, pl->q_slots, pl->p_bufs, pl->box_tokens,
                                      pl->smem_bytes, fused, pl->withhold_tile, stream);
  } else {
    ce = lse_launch_partial_cuda_core(p, pl->dtype, pl->head_dim, pl->n_splits, pl->n_kv_heads,
                                      pl->n_seqs, pl->smem_bytes, stream);
  }
  if (ce) return cuda_fail(err, ce, "partial kernel launch");
  return LSE_OK;
}

int lse_attn_run(const lse_attn_plan_t *pl, const float *q, const int32_t *k_pages,
                 const int32_t *v_pages, const int32_t *seq_lens, const int32_t *row_offsets,
                 const uint64_t *row_masks, float softmax_scale, void *ws, void *stream,
                 char **err) {
  return launch_partial(pl, q, k_pages, v_pages, seq_lens, row_offsets, row_masks,
                        softmax_scale, ws, nullptr, nullptr, 0, stream, err);
}

int lse_attn_forward(const lse_attn_plan_t *pl, const float *q, const int32_t *k_pages,
                     const int32_t *v_pages, const int32_t *seq_lens, const int32_t *row_offsets,
                     const uint64_t *row_masks, float softmax_scale, void *ws, float *out,
                     float *lse_out, void *stream, char **err) {
  if (!pl) return fail(err, LSE_ERR_INVALID_ARG, "plan is NULL");
  if (!out) return fail(err, LSE_ERR_INVALID_ARG, "out is NULL");
  if (pl->kernel != LSE_KERNEL_CUDA_CORE)
    return launch_partial(pl, q, k_pages, v_pages, seq_lens, row_offsets, row_masks,
                          softmax_scale, ws, out, lse_out, 1, stream, err);
  const int st = launch_partial(pl, q, k_pages, v_pages, seq_lens, row_offsets, row_masks,
                                softmax_scale, ws, nullptr, nullptr, 0, stream, err);
  if (st) return st;
  return lse_attn_merge(pl, seq_lens, row_offsets, ws, out, lse_out, stream, err);
}

int lse_attn_merge(const lse_attn_plan_t *pl, const int32_t *seq_lens, const int32_t *row_offsets,
                   const void *ws, float *out, float *lse_out, void *stream, char **err) {
  if (!pl) return fail(err, LSE_ERR_INVALID_ARG, "plan is NULL");
  if (pl->kernel == LSE_KERNEL_PREFILL)
    return fail(err, LSE_ERR_UNSUPPORTED, "a long-query-block plan runs through "
                "lse_attn_forward");
  if (!seq_lens || !row_offsets || !ws || !out)
    return fail(err, LSE_ERR_INVALID_ARG, "a required device pointer is NULL");
  LseKernelParams p;
  int st = fill_params(pl, const_cast<void *>(ws), p, err);
  if (st) return st;
  p.seq_lens = seq_lens;
  p.row_offsets = row_offsets;
  p.balanced = pl->kernel == LSE_KERNEL_TCGEN05;
  p.n_ctas = pl->ctas;
  p.out = out;
  p.lse_out = lse_out;
  int ce = lse_launch_merge(p, pl->head_dim, stream);
  if (ce) return cuda_fail(err, ce, "merge kernel launch");
  return LSE_OK;
}

int lse_attn_read_error(const lse_attn_plan_t *pl, void *ws, void *stream, uint32_t *device_error,
                        char **err) {
  if (!pl || !ws || !device_error)
    return fail(err, LSE_ERR_INVALID_ARG, "plan, workspace or result is NULL");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  int ce = (int)cudaMemcpyAsync(&v, ws, sizeof v, cudaMemcpyDeviceToHost, st);
  if (!ce) ce = (int)cudaStreamSynchronize(st);
  // after a fault the fused merge's segment counters may be left part-way:
  // clear them with the error word
  if (!ce) ce = (int)cudaMemsetAsync(ws, 0, v ? pl->ws_o_off : sizeof v, st);
  if (ce) return cuda_fail(err, ce, "reading the device error word");
  *device_error = v;
  return LSE_OK;
}

// ---- validation of host copies --------------------------------------------------

int lse_attn_validate(const lse_attn_plan_t *pl, const int32_t *k_pages, const int32_t *v_pages,
                      const int32_t *seq_lens, const int32_t *row_offsets,
                      const uint64_t *row_masks, char **err) {
  if (!pl || !k_pages || !v_pages || !seq_lens || !row_offsets)
    return fail(err, LSE_ERR_INVALID_ARG, "a required host pointer is NULL");
  const lse_kv_arena *a = pl->arena;
  const int32_t n_frag = int32_t(a->used.size());
  const int64_t T = a->tokens_per_fragment;
  const int64_t cap = int64_t(pl->max_pages) * T;
  if (row_offsets[0] != 0) return fail(err, LSE_ERR_BAD_INPUT, "row_offsets[0] != 0");
  for (int s = 0; s < pl->n_seqs; ++s) {
    const int64_t L = seq_lens[s];
    const int R = row_offsets[s + 1] - row_offsets[s];
    if (R < 0 || R > pl->max_rows)
      return fail(err, LSE_ERR_BAD_INPUT, "sequence %d: %d rows (max %d)", s, R, pl->max_rows);
    if (L < 0 || L > cap)
      return fail(err, LSE_ERR_BAD_INPUT, "sequence %d: length %lld beyond capacity %lld", s,
                  (long long)L, (long long)cap);
    if (R > L) return fail(err, LSE_ERR_BAD_INPUT, "sequence %d: %d rows > %lld keys", s, R,
                           (long long)L);
    const int64_t pages = (L + T - 1) / T;
    for (int which = 0; which < 2; ++which) {
      const int32_t *tab = which ? v_pages : k_pages;
      for (int64_t pg = 0; pg < pages; ++pg) {
        const int32_t f = tab[int64_t(s) * pl->max_pages + pg];
        if (f < 0 || f >= n_frag)
          return fail(err, LSE_ERR_BAD_INPUT, "sequence %d %s page %lld: fragment %d unknown",
                      s, which ? "V" : "K", (long long)pg, f);
      }
    }
    if (row_masks && R > LSE_MAX_ROWS_PER_SEQ)
      return fail(err, LSE_ERR_BAD_INPUT, "sequence %d: %d rows with masks (masks take at "
                  "most %d rows)", s, R, LSE_MAX_ROWS_PER_SEQ);
    for (int r = 0; r < R && row_masks; ++r) {
      const uint64_t m = row_masks[row_offsets[s] + r];
      if (!((m >> r) & 1u))
        return fail(err, LSE_ERR_BAD_INPUT, "sequence %d row %d: mask misses itself", s, r);
      if (r < 63 && (m >> (r + 1)))
        return fail(err, LSE_ERR_BAD_INPUT, "sequence %d row %d: mask names a later row", s,
                    r);
    }
  }
  if (row_offsets[pl->n_seqs] > pl->max_total_rows)
    return fail(err, LSE_ERR_BAD_INPUT, "%d rows exceed max_total_rows %d",
                row_offsets[pl->n_seqs], pl->max_total_rows);
  return LSE_OK;
}

}  // extern "C"
