// Tensor-core prefill path (tcgen05, bf16 operands, dk = dv = 128).
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "kda_internal.h"

// Status word value recorded by a kernel whose bounded wait gave up
// (the value of KDA_ERR_TIMEOUT in include/kda.h).
#define KDA_TC_TIMEOUT_CODE 5

namespace kda {

// Segments per sequence of the split plan (1 = no split): 2 G - 1 state CTAs
// per (sequence, head) must fit on the 148 SMs, and, unless `forced`, every
// segment must keep 16 chunks of 64 tokens on average.  `forced` gives G >= 2.
int tc_split_segments(int32_t total_tokens, int32_t num_seqs, int32_t H, bool forced);

// Workspace bytes of the tensor-core path: the chunk plan plus one 74,496-byte
// block of MMA-ready tiles per (chunk, head), for the worst case of
// floor((T + 63 N) / 64) chunks; with segments > 1 also the segment states,
// transitions, S_in images (N G H of each) and 16 KiB E images per (chunk, head).
// With gate == 1 (the unbounded Softplus gate) it also holds the pair kernel's
// diagonal tiles, 8 KiB per (chunk, head).
size_t tc_workspace_bytes(int32_t total_tokens, int32_t num_seqs, int32_t H, int segments,
                          int gate = 0);

// Launches plan, intra-chunk and state kernels on `stream`, then, when
// a.segments > 1, the segment composition and the output correction.
cudaError_t launch_prefill_tensor_core(const PrefillArgs &a, cudaStream_t stream);

}  // namespace kda
