// Internal declarations shared by the host side (lse_host.cpp) and the
// kernels (lse_kernels.cu) of liblse_attn.so.  Not part of the C ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <mutex>
#include <string>
#include <vector>

#include "lse_attn.h"

struct lse_kv_arena {
  std::vector<uint64_t> chunk_base;  // device addresses
  size_t chunk_bytes = 0;
  size_t fragment_bytes = 0;
  int dtype = 0;
  int n_kv_heads = 0;
  int head_dim = 0;
  int esize = 0;
  int tokens_per_fragment = 0;
  int frags_per_chunk = 0;
  std::vector<uint8_t> used;        // per fragment id
  std::vector<int32_t> chunk_live;  // live fragments per chunk
  int32_t n_free = 0;
  int32_t scan_from = 0;            // lowest id that may be free
  float *scales = nullptr;          // per-vector scales by fragment (device), or null
  int64_t n_scales = 0;             // floats in scales
};

struct lse_attn_plan_s {
  const lse_kv_arena *arena = nullptr;
  int n_seqs = 0;
  int max_rows = 0;
  int max_total_rows = 0;
  int n_q_heads = 0;
  int n_kv_heads = 0;
  int group = 0;        // G = Hq / Hkv
  int head_dim = 0;
  int dtype = 0;
  int max_pages = 0;
  int tokens_per_fragment = 0;
  int n_splits = 0;
  int keys_per_split = 0;
  int kernel = 0;
  int key_tile = 0;
  int pairs = 0;        // G * max_rows
  int smem_bytes = 0;
  int n_sms = 0;
  int ctas = 0;          // persistent grid of the tensor-core kernel
  int stages = 0;        // its K ring depth (prefill: the K/V ring depth)
  int v_stages = 0;      // its V ring depth
  int q_slots = 0;       // and its Q ring depth
  int p_bufs = 0;        // and its P tiles per softmax group
  int pairs_bucket = 0;  // its compile-time pair count (P8)
  int rows_per_chunk = 0;  // tensor-core kernel: query rows per segment
  int box_tokens = 0;    // its TMA box height
  int scaled = 0;        // made for an arena with per-vector scales
  int withhold_tile = -1;  // tests of the bounded waits (lse_attn_test_withhold_tile)
  // tensor maps of the arena chunks (built on first run, rebuilt on growth);
  // maps_mutex guards them, so threads may run one plan at the same time
  mutable std::vector<uint8_t> maps;
  mutable int maps_chunks = 0;
  mutable std::mutex maps_mutex;
  size_t ws_bytes = 0;
  size_t ws_cnt_off = 0; // tensor-core kernel: per-segment counters of the fused merge
  int n_seg_max = 0;     //   (two uint32 per segment), zeroed by lse_attn_workspace_init
  size_t ws_o_off = 0;   // partial outputs  FP32 [rows][Hq][n_splits][D]
  size_t ws_lse_off = 0; // partial lse (log2 units) FP32 [rows][Hq][n_splits]
};

// Bytes reserved at the head of the workspace (error word + padding).
constexpr size_t kWsHeader = 256;

// Cut of the tensor-core pass's live tiles into CTA ranges, shared by the
// pass and the separate merge (which counts each segment's pieces): every
// segment counts kLseSegWeight tiles more than it has, when the call has at
// most kLseSeqTab sequences (the pass keeps them in a shared-memory table)
// and each working CTA's share is at least kLseSegMinShare tiles.
constexpr int kLseSeqTab = 96;
constexpr int kLseSegWeight = 5;
constexpr int kLseSegMinShare = 8 * kLseSegWeight;

// Parameters passed by value to the partial and merge kernels.
struct LseKernelParams {
  unsigned long long chunk_base[LSE_MAX_CHUNKS];
  long long fragment_bytes;
  int frags_per_chunk;
  int n_fragments;
  int n_q_heads;
  int n_kv_heads;
  int group;
  int head_dim;
  int tokens_per_fragment;
  int max_pages;
  int n_splits;
  int keys_per_split;
  int max_rows;
  int max_total_rows;
  int n_seqs;
  float scale_log2;  // softmax_scale * log2(e)
  const float *q;
  const int32_t *k_pages;
  const int32_t *v_pages;
  const int32_t *seq_lens;
  const int32_t *row_offsets;
  const unsigned long long *row_masks;
  float *o_part;
  float *lse_part;
  unsigned int *err;
  float *out;
  float *lse_out;
  int rows_per_chunk;  // tcgen05: query rows per segment (row chunk)
  int balanced;    // merge: 1 = slots are persistent-CTA pieces (tcgen05)
  int n_ctas;      // persistent grid size when balanced
  // per-vector scales: a [kv_head][token] FP32 block per fragment id, or
  // null for unit scales
  const float *scales;
  // tensor-core kernel with the merge fused: two counters per segment
  unsigned int *seg_count;
};

// Arguments of the K/V append kernel (lse_append.cu).
struct AppendParams {
  unsigned long long chunk_base[LSE_MAX_CHUNKS];
  long long fragment_bytes;
  int frags_per_chunk;
  int n_fragments;
  int tokens_per_fragment;
  int n_kv_heads;
  int n_seqs;
  int max_pages;
  int total_new;
  const float *k_new;
  const float *v_new;
  const int32_t *k_pages;
  const int32_t *v_pages;
  const int32_t *seq_lens_before;
  const int32_t *new_offsets;
  unsigned int *err;
  float *scales;  // 8-bit arenas with per-vector scales: written with the vectors
};
int lse_launch_kv_append(const AppendParams &a, int dtype, int head_dim, void *stream);

// Kernel entry points (lse_kernels.cu).  Return a cudaError_t value.
int lse_launch_partial_cuda_core(const LseKernelParams &p, int dtype, int head_dim, int grid_x,
                                 int grid_y, int grid_z, int smem, void *stream);
int lse_launch_merge(const LseKernelParams &p, int head_dim, void *stream);
int lse_partial_cuda_core_smem(int head_dim);
int lse_partial_cuda_core_occupancy(int dtype, int head_dim, int smem, int *ctas_per_sm);
const char *lse_cuda_error_string(int code);

// tensor-core partial pass (lse_tcgen05.cu)
int lse_tc_pairs_bucket(int pairs);
int lse_tc_smem(int dtype, int p8, int scaled, int smem_optin, int *k_stages, int *v_stages,
                int *q_slots, int *p_bufs);
int lse_tc_key_tile();
size_t lse_tc_map_bytes();
int lse_tc_build_maps(const uint64_t *chunk_base, int n_chunks, size_t chunk_bytes,
                      int n_kv_heads, int dtype, int box_tokens, void *maps_out);
int lse_launch_partial_tcgen05(const LseKernelParams &p, const void *maps, int n_maps,
                               int dtype, int p8, int scaled, int n_ctas, int n_slots,
                               int k_stages, int v_stages, int q_slots, int p_bufs,
                               int box_tokens, int smem, int fused, int withhold_tile,
                               void *stream);
// long query blocks (lse_prefill.cu)
int lse_pf_row_tile();
int lse_pf_max_row_tiles();
int lse_pf_smem(int dtype, int smem_optin, int *stages);
int lse_launch_prefill_tcgen05(const LseKernelParams &p, const void *maps, int n_maps, int dtype,
                               int n_ctas, int stages, int box_tokens, int smem, void *stream);
