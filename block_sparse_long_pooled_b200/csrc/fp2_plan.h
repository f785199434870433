// Host-computed launch plan shared by every kernel of the library.
//
// The host owns the authoritative sequence lengths (fp2_problem.cu_seqlens_*_host),
// so it builds this table once per call and passes it by value as a kernel
// parameter: no device-side planning kernel, nothing to copy, and nothing a
// stream capture cannot record.
#pragma once

#include <stdint.h>

#include "../../include/fp2.h"

// Queries of sequence r are its last len[r] tokens (the whole sequence, or a chunk at its end);
// its keys are pre_blk[r] * B + len[r] tokens, and query block i is absolute key block
// pre_blk[r] + i.  At FP2_MAX_SEQS = 512 the table is ~20 KB, so kernels take it as a
// __grid_constant__ parameter (read in place, never copied) and rely on the 32 KB kernel-parameter
// limit of CUDA 12.1 and later.
struct Fp2Plan {
  int32_t num_seqs;
  int32_t total_tokens;             // query tokens
  int32_t total_blocks;             // query blocks
  int32_t total_k_tokens;
  int32_t total_k_blocks;
  int32_t max_nblk;                 // most query blocks of any sequence
  int32_t max_k_nblk;               // most key blocks of any sequence
  int32_t disc_tile;                // query blocks per discovery CTA (the tile of lvl_base_t)
  int32_t tok_off[FP2_MAX_SEQS];    // first query token of sequence r in Q
  int32_t len[FP2_MAX_SEQS];        // query tokens L_r
  int32_t blk_off[FP2_MAX_SEQS];    // first query block of sequence r
  int32_t nblk[FP2_MAX_SEQS];       // query blocks N_r = ceil(L_r / B)
  int32_t k_tok_off[FP2_MAX_SEQS];  // first key token of sequence r in contiguous K/V
  int32_t k_blk_off[FP2_MAX_SEQS];  // first key block of sequence r (pooled kbar/vbar rows)
  int32_t pre_blk[FP2_MAX_SEQS];    // key blocks before the query chunk
  int16_t sorted[FP2_MAX_SEQS];     // sequence ids by N_r descending (heavy rows first)
  // Heavy-first work lists (fp2_device.cuh, map_heavy_first): with the sequences in `sorted`
  // order and hi_k = levels of the k-th (ceil(nblk / tile)), lo_k = those of the (k+1)-th,
  // lvl_base[k] = sum_{k' < k} (hi_k' - lo_k') * (k' + 1) items per unit of width.  lvl_base1 is
  // for a tile of one query block (pool order, attention), lvl_base_t for disc_tile.
  int32_t lvl_base1[FP2_MAX_SEQS + 1];
  int32_t lvl_base_t[FP2_MAX_SEQS + 1];
};

// Device status bits live in the first word of scratch.
#define FP2_SCRATCH_STATUS_BYTES 256
