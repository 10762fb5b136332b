// Tensor-core prefill path (tcgen05, bf16 operands, dk = dv = 128).
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "kda_internal.h"

// Status word value recorded by a kernel whose bounded wait gave up
// (the value of KDA_ERR_TIMEOUT in include/kda.h).
#define KDA_TC_TIMEOUT_CODE 5

namespace kda {

// Workspace bytes of the tensor-core path: the chunk plan plus one 74,240-byte
// block of MMA-ready tiles per (chunk, head), for the worst case of
// floor((T + 63 N) / 64) chunks.
size_t tc_workspace_bytes(int32_t total_tokens, int32_t num_seqs, int32_t H);

// Launches plan, intra-chunk and state kernels on `stream`.
cudaError_t launch_prefill_tensor_core(const PrefillArgs &a, cudaStream_t stream);

}  // namespace kda
