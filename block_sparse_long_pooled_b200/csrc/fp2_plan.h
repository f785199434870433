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
// pre_blk[r] + i.  The table is ~3.8 KB, so kernels taking it rely on the kernel-parameter limit
// of 32 KB (CUDA 12.1 and later).
struct Fp2Plan {
  int32_t num_seqs;
  int32_t total_tokens;             // query tokens
  int32_t total_blocks;             // query blocks
  int32_t total_k_tokens;
  int32_t total_k_blocks;
  int32_t max_nblk;                 // most query blocks of any sequence
  int32_t max_k_nblk;               // most key blocks of any sequence
  int32_t tok_off[FP2_MAX_SEQS];    // first query token of sequence r in Q
  int32_t len[FP2_MAX_SEQS];        // query tokens L_r
  int32_t blk_off[FP2_MAX_SEQS];    // first query block of sequence r
  int32_t nblk[FP2_MAX_SEQS];       // query blocks N_r = ceil(L_r / B)
  int32_t k_tok_off[FP2_MAX_SEQS];  // first key token of sequence r in contiguous K/V
  int32_t k_blk_off[FP2_MAX_SEQS];  // first key block of sequence r (pooled kbar/vbar rows)
  int32_t pre_blk[FP2_MAX_SEQS];    // key blocks before the query chunk
  int16_t sorted[FP2_MAX_SEQS];     // sequence ids by N_r descending (heavy rows first)
};

// Device status bits live in the first word of scratch.
#define FP2_SCRATCH_STATUS_BYTES 256
