// Host-computed launch plan shared by every kernel of the library.
//
// The host owns the authoritative sequence lengths (fp2_problem.cu_seqlens_*_host),
// so it builds this table once per call and passes it by value as a kernel
// parameter: no device-side planning kernel, nothing to copy, and nothing a
// stream capture cannot record.
#pragma once

#include <stdint.h>

#include "../../include/fp2.h"

struct Fp2Plan {
  int32_t num_seqs;
  int32_t total_tokens;
  int32_t total_blocks;
  int32_t max_nblk;
  int32_t tok_off[FP2_MAX_SEQS];  // first token of sequence r in the packed batch
  int32_t len[FP2_MAX_SEQS];      // L_r
  int32_t blk_off[FP2_MAX_SEQS];  // first pooled block of sequence r
  int32_t nblk[FP2_MAX_SEQS];     // N_r = ceil(L_r / B)
  int16_t sorted[FP2_MAX_SEQS];   // sequence ids by N_r descending (heavy rows first)
};

// Device status bits live in the first word of scratch.
#define FP2_SCRATCH_STATUS_BYTES 256
