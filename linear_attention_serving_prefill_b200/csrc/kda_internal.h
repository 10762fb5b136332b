// Internal launch interface between the C-ABI layer (kda_api.cu) and the kernel
// translation units.  Every launcher enqueues on `stream` and returns the
// cudaGetLastError() of its launch.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

// Identifier of the calling thread's current CUDA context (cuCtxGetId: unique
// for the process lifetime, so a context destroyed and created again, as by
// cudaDeviceReset, gets a new one).  False when no context is current.
bool current_context_id(unsigned long long *id);

struct PrefillArgs {
    const void *q, *k, *v, *z;
    const float *A, *beta;
    const int32_t *cu_seqlens;      // device [N+1]
    const int32_t *seq_order;       // device [N] launch order (longest first) or nullptr
    int32_t num_seqs, total_tokens, H, dk, dv;
    bool bf16;                      // storage dtype of q, k, v, z, o
    const float *initial_state;     // [N,H,dk,dv] or nullptr
    float *final_state;             // [N,H,dk,dv] or nullptr
    void *o;
    void *workspace;
    size_t workspace_bytes;
    int32_t *status;                // device status word
    int32_t ckpt_every;             // 0 = no checkpoints, else a multiple of 64
    float *checkpoints;             // [count, H, dk, dv] or nullptr
    int32_t segments;               // tensor-core path: segments per sequence (1 = no split)
    int32_t gate = 0;               // 0 = K3 lower-bounded gate, 1 = unbounded -softplus
    // Debug dumps of the tensor-core path's stages (fp32 [T, H, 128]; nullptr = none).
    float *dbg_G = nullptr, *dbg_W = nullptr, *dbg_U = nullptr, *dbg_delta = nullptr;
    void *const *events;            // optional cudaEvent_t per kernel boundary
    int32_t num_events;
    // Records boundary i (0 = before the first kernel) when the caller asked for it.
    void mark(int i, cudaStream_t stream) const {
        if (events && i < num_events && events[i]) cudaEventRecord((cudaEvent_t)events[i], stream);
    }
};

struct DecodeArgs {
    const void *q, *k, *v, *z;
    const float *A, *beta;
    int32_t B, H, dk, dv;
    bool bf16;
    float *state;
    const int32_t *slots;
    void *o;
    int32_t gate = 0;               // as PrefillArgs::gate
};

struct DecodeMultiArgs {
    const void *q, *k, *v, *z;      // [B, Tq, H, d]
    const float *A, *beta;          // beta [B, Tq, H]
    int32_t B, Tq, H, dk, dv;
    bool bf16;
    float *state;
    const int32_t *slots;
    const int32_t *num_tokens;      // [B] or nullptr (= Tq)
    bool update_state;
    void *o;                        // [B, Tq, H, dv] or nullptr
    int32_t *status;                // device status word (a wait that gives up records here)
};

// Tq tokens per sequence on a register-resident state (verify / replay).
cudaError_t launch_decode_multi(const DecodeMultiArgs &a, cudaStream_t stream);

// Fused chunked prefill on CUDA cores, all arithmetic in fp32 (16-token chunks).
cudaError_t launch_prefill_cuda_core(const PrefillArgs &a, cudaStream_t stream);

// One-CTA kernel whose bounded mbarrier wait is never satisfied (records a timeout).
cudaError_t launch_wait_timeout_selftest(int32_t *status, int64_t limit_ns, cudaStream_t stream);

// Single-token decode step (HBM-bound, one CTA per (sequence, head)).
cudaError_t launch_decode_step(const DecodeArgs &a, cudaStream_t stream);

}  // namespace kda
