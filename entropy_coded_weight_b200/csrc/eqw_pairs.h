// Host entry of the pair decode kernel (eqw_decode_pairs.cu), used by the
// decode launcher in eqw_decode.cu.
#pragma once

#include <cuda_runtime.h>

#include "eqw_internal.h"

namespace eqw {

// True if matrix d written to `out` can go through the pair kernel: one
// frequency table for all chunks with 2..32 symbols, rows a multiple of 512
// symbols, 16-byte aligned output, at least one pair of full chunks.
bool pair_eligible(const MatrixDesc &d, const void *out);

// Decode, for each eligible matrix mats[i] (output outs[i]), its leading pairs
// of full chunks; handled[i] receives the number of leading chunks decoded (0
// for a matrix left entirely to the caller).  Launches on stream s, at most
// one block per SM of `sms`.
int launch_decode_pairs(const eq_model *m, const uint32_t *mats, uint16_t *const *outs, uint32_t count,
                        int32_t *d_status, cudaStream_t s, int sms, uint32_t *handled);

// Host-only form of the same decision: handled[i] = leading chunks of mats[i]
// the pair kernel would decode on `sms` SMs (outputs 256-byte aligned).
int plan_decode_pairs(const eq_model *m, const uint32_t *mats, uint32_t count, uint32_t sms, uint32_t *handled);

}  // namespace eqw
