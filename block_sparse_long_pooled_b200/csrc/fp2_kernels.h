// Kernel argument blocks and launchers (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fp2_plan.h"

namespace fp2 {

struct PoolArgs {
  const void* q;
  const void* k;
  const void* v;
  int64_t q_stride, kv_stride;  // elements between tokens
  const int32_t* page_table;    // NULL -> contiguous K/V
  int page_size, max_pages, num_pages;
  int Hq, Hkv, D, B;
  float q_descale, k_descale, v_descale;
  float* qbar;
  float* kbar;
  float* vbar;
  void* kbar_mma;
  void* vbar_mma;
  void* v16;             // E4M3: f16 copy of V in key-token order (NULL otherwise)
  int kv_prefix_pooled;  // skip K/V of prefix blocks (already pooled)
  uint32_t* status;
};

struct DiscArgs {
  const float* qbar;
  const float* kbar;
  int Hq, Hkv, G, D;
  float scale;      // softmax scale used for the block scores
  float ln_alpha;   // natural log of alpha (alpha > 0)
  int dense_all;    // alpha <= 0: keep everything
  int sink, window, last_n, min_sparse_len;
  int TI;           // query blocks per CTA: 128 / G (the CTA's 128 score rows)
  int W;            // bitmask words per row
  uint32_t* bitmask;
  int32_t* counts;
  uint32_t* status;
};

struct AttnArgs {
  CUtensorMap tm_q;   // Q  [T, Hq, d]       box {128B / elt, 1, B}
  CUtensorMap tm_k;   // K  tokens (flat)    box {128B / elt, 1, B or page rows}
  CUtensorMap tm_v;   // V, or for E4M3 inputs its f16 copy [Tk, Hkv, d] (contiguous, box {64, 1, B})
  CUtensorMap tm_kb;  // kbar_mma [blocks, Hkv, d] box {128B / elt, 1, B}
  CUtensorMap tm_vb;
  CUtensorMap tm_o;   // out [T, Hq, d] (bf16, or f32 for f32 inputs) box {128B / elt, 1, B}
  int o_tma;          // 1: full blocks are written through tm_o by TMA stores
  int v_contig;       // 1: V tiles come from tm_v's contiguous rows even when K is paged (E4M3)
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const int32_t* page_table;  // NULL -> contiguous
  int page_size, max_pages, num_pages;
  void* out;                  // [T, Hq, d] bf16 (f32 for f32 inputs)
  float* lse;                 // [Hq, T] or NULL
  int Hq, Hkv, G;
  int NT;                     // M tiles (128 packed rows each) per CTA: 1 or 2
  int parts;                  // CTAs per (sequence, query block, KV head)
  float sm_scale_log2;        // softmax scale * log2(e) * q_descale * k_descale
  float v_descale;
  float log2_blk;             // log2 of a pruned block's token count
  int mean_correction;
  int total_tokens;
  int splits;                 // KV splits per row (1 = none)
  int num_sms;                // SMs of the device (the launch's wave width)
  float* o_part;              // [splits, T, Hq, d] f32 partial outputs (splits > 1)
  float* lse_part;            // [splits, Hq, T] f32 partial LSE (splits > 1)
  // Adaptive splits: CTAs [0, adapt) of the launch run the pieces listed by split_plan_kernel;
  // the rows those pieces cover are skipped by their own CTAs.  adapt = 0: none.
  int adapt;                  // piece capacity (CTAs launched ahead of the row CTAs)
  int32_t* row_item0;         // [rows] first piece of the row, or -1 when the row is not split
  int2* items;                // [adapt] piece: {row, (pieces of the row << 16) | (part << 8) | piece}
  int32_t* n_items;           // pieces planned (<= adapt)
  int32_t* piece_cnt;         // [adapt * 2] finished pieces per (first piece of a row part, M tile)
  float* o_slot;              // [adapt, NT * 128, d] f32 normalised partial outputs of the pieces
  float* lse_slot;            // [adapt, NT * 128] f32 natural-log partial LSE
  uint32_t* status;
  uint64_t wait_limit_ns;     // limit of every mbarrier wait (drains of in-flight copies: a fifth)
  int withhold_k_tile;        // testing: the producer skips the K load of this local key tile (-1: none)
  int miscount_load;          // testing, checked builds: the producer counts this load twice (-1: none)
};

// Raise a kernel's dynamic shared-memory limit to at least `bytes` on the current device.  The
// attribute call is made only when the limit grows (it is slow enough to starve the GPU when a
// caller issues many short launches, e.g. one per prefill chunk).
cudaError_t ensure_dynamic_smem(const void* kernel, int bytes);

cudaError_t launch_pool(int dtype, const PoolArgs& a, const Fp2Plan& P, cudaStream_t stream);
size_t discover_smem_bytes(int D);
cudaError_t launch_discover(const DiscArgs& a, const Fp2Plan& P, int64_t items, int64_t rows, int32_t* row_ptr,
                            int32_t* col_idx, int64_t capacity, cudaStream_t stream);
// Returns cudaErrorInvalidValue when no kernel exists for (dtype, d, B).
cudaError_t launch_attention(int dtype, int D, int B, const AttnArgs& a, const Fp2Plan& P, int64_t items,
                             cudaStream_t stream);
size_t attention_smem_bytes(int dtype, int D, int B);
// Plans the adaptive pieces of one attention launch from the index's row_ptr (a.adapt > 0):
// piece_tiles > 0 cuts rows longer than that many key tiles; 0 derives the size from the launch.
cudaError_t launch_split_plan(const AttnArgs& a, const Fp2Plan& P, int64_t rows, int B, int piece_tiles,
                              cudaStream_t stream);
cudaError_t launch_combine(int dtype, int D, const float* o_part, const float* lse_part, int S, int T, int Hq,
                           void* out, float* lse, cudaStream_t stream);

}  // namespace fp2
