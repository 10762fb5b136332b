// C-ABI layer of libkda_b200: argument validation, workspace sizing and
// dispatch to the kernels.  Nothing here allocates device memory; every call is
// asynchronous on the caller's stream.
#include <cuda.h>
#include <mutex>
#include <vector>
#include <stdint.h>
#include <string.h>

#include "kda.h"
#include "kda_internal.h"
#include "kda_prefill_tc.h"

// Device status word: kernels with bounded on-chip waits record a timeout here
// instead of hanging.  One instance per device that loads the library.
__device__ int32_t g_kda_device_status = 0;

namespace kda {

// cuCtxGetCurrent / cuCtxGetId, fetched from the driver through the runtime (no
// link-time dependency on libcuda).
bool current_context_id(unsigned long long *id)
{
    using GetCurrent = CUresult (*)(CUcontext *);
    using GetId = CUresult (*)(CUcontext, unsigned long long *);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = (GetCurrent)p;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = (GetId)p;
    });
    CUcontext ctx = nullptr;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

}  // namespace kda

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_status_mu;
// Per device: the status word's device address and the context it belongs to.
// A device reset destroys the context (and unloads the module); the next call
// sees a new context id and looks the address up again.
int32_t *g_status_ptr[kMaxDevices] = {nullptr};
unsigned long long g_status_ctx[kMaxDevices] = {0};

bool head_dim_ok(int32_t d) { return d == 32 || d == 64 || d == 128; }
bool aligned(const void *p, uintptr_t a) { return ((uintptr_t)p % a) == 0; }

kda_status status_word(int32_t **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KDA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_status_mu);
    unsigned long long ctx = 0;
    const bool have_ctx = kda::current_context_id(&ctx);
    if (!g_status_ptr[dev] || !have_ctx || ctx != g_status_ctx[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_kda_device_status) != cudaSuccess) return KDA_ERR_CUDA;
        g_status_ptr[dev] = (int32_t *)p;
        // The lookup made the device's primary context current if it was not.
        g_status_ctx[dev] = kda::current_context_id(&ctx) ? ctx : 0;
    }
    *out = g_status_ptr[dev];
    return KDA_OK;
}

// Validation shared by kda_prefill_workspace_size and kda_prefill_ex.
kda_status check_prefill_sizes(int32_t total_tokens, int32_t num_seqs, int32_t H, int32_t dk,
                               int32_t dv, kda_dtype dt, kda_algo algo)
{
    if (total_tokens < 0 || num_seqs < 0 || H <= 0) return KDA_ERR_INVALID_ARG;
    if (dt != KDA_DTYPE_BF16 && dt != KDA_DTYPE_F32) return KDA_ERR_INVALID_ARG;
    if (algo != KDA_ALGO_AUTO && algo != KDA_ALGO_CUDA_CORE && algo != KDA_ALGO_TENSOR_CORE &&
        algo != KDA_ALGO_TENSOR_CORE_SPLIT)
        return KDA_ERR_INVALID_ARG;
    if (dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if ((algo == KDA_ALGO_TENSOR_CORE || algo == KDA_ALGO_TENSOR_CORE_SPLIT) &&
        (dt != KDA_DTYPE_BF16 || dk != 128 || dv != 128))
        return KDA_ERR_UNSUPPORTED;
    return KDA_OK;
}

// The path a call takes: tensor cores for bf16 with dk = dv = 128 unless the
// CUDA-core path is forced; the fp32 CUDA-core path otherwise.
bool use_tensor_core(int32_t dk, int32_t dv, kda_dtype dt, kda_algo algo)
{
    if (algo == KDA_ALGO_TENSOR_CORE || algo == KDA_ALGO_TENSOR_CORE_SPLIT) return true;
    if (algo == KDA_ALGO_CUDA_CORE) return false;
    return dt == KDA_DTYPE_BF16 && dk == 128 && dv == 128;
}

// Segments per sequence on the tensor-core path: AUTO splits when few
// (sequence, head) chains would leave most SMs idle, SPLIT always does,
// TENSOR_CORE never.  (Valid arguments assumed.)
int32_t segments_for(int32_t total_tokens, int32_t num_seqs, int32_t H, int32_t dk, int32_t dv,
                     kda_dtype dt, kda_algo algo)
{
    if (!use_tensor_core(dk, dv, dt, algo) || algo == KDA_ALGO_TENSOR_CORE) return 1;
    return kda::tc_split_segments(total_tokens, num_seqs, H, algo == KDA_ALGO_TENSOR_CORE_SPLIT);
}

}  // namespace

extern "C" int32_t kda_abi_version(void) { return KDA_ABI_VERSION; }

extern "C" const char *kda_status_string(kda_status s)
{
    switch (s) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG: invalid argument";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: unsupported configuration";
    case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE: workspace missing or too small";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA: CUDA runtime error";
    case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT: an on-device wait gave up";
    }
    return "KDA_ERR_UNKNOWN";
}

extern "C" size_t kda_prefill_gated_workspace_size(int32_t total_tokens, int32_t num_seqs,
                                                   int32_t H, int32_t dk, int32_t dv, kda_dtype dt,
                                                   kda_algo algo, kda_gate gate)
{
    if (check_prefill_sizes(total_tokens, num_seqs, H, dk, dv, dt, algo) != KDA_OK) return 0;
    if (gate != KDA_GATE_LOWER_BOUNDED && gate != KDA_GATE_SOFTPLUS) return 0;
    if (use_tensor_core(dk, dv, dt, algo))
        return kda::tc_workspace_bytes(total_tokens, num_seqs, H,
                                       segments_for(total_tokens, num_seqs, H, dk, dv, dt, algo),
                                       gate == KDA_GATE_SOFTPLUS ? 1 : 0);
    return 0;  // the CUDA-core path keeps everything on chip
}

extern "C" size_t kda_prefill_workspace_size(int32_t total_tokens, int32_t num_seqs, int32_t H,
                                             int32_t dk, int32_t dv, kda_dtype dt, kda_algo algo)
{
    return kda_prefill_gated_workspace_size(total_tokens, num_seqs, H, dk, dv, dt, algo,
                                            KDA_GATE_LOWER_BOUNDED);
}

extern "C" int32_t kda_prefill_segments(int32_t total_tokens, int32_t num_seqs, int32_t H,
                                        int32_t dk, int32_t dv, kda_dtype dt, kda_algo algo)
{
    if (check_prefill_sizes(total_tokens, num_seqs, H, dk, dv, dt, algo) != KDA_OK) return 0;
    return segments_for(total_tokens, num_seqs, H, dk, dv, dt, algo);
}

extern "C" int64_t kda_checkpoint_count(const int32_t *cu_seqlens_host, int32_t num_seqs,
                                        int32_t checkpoint_every)
{
    if (num_seqs < 0 || checkpoint_every <= 0 || checkpoint_every % 64 != 0) return -1;
    if (num_seqs > 0 && !cu_seqlens_host) return -1;
    int64_t total = 0;
    for (int32_t i = 0; i < num_seqs; ++i) {
        const int32_t L = cu_seqlens_host[i + 1] - cu_seqlens_host[i];
        if (L < 0) return -1;
        total += L / checkpoint_every;
    }
    return total;
}

namespace {

// Every prefill entry point lands here.
kda_status prefill_impl(const void *q, const void *k, const void *v, const void *z, const float *A,
                        const float *beta, const int32_t *cu_seqlens_dev,
                        const int32_t *cu_seqlens_host, int32_t num_seqs, int32_t total_tokens,
                        int32_t H, int32_t dk, int32_t dv, kda_dtype dt,
                        const float *initial_state, float *final_state, void *o, void *workspace,
                        size_t workspace_bytes, kda_algo algo, void *stream,
                        void *const *stage_events, int32_t num_stage_events,
                        int32_t checkpoint_every, float *checkpoints, kda_gate gate,
                        float *const *dbg = nullptr)
{
    kda_status st = check_prefill_sizes(total_tokens, num_seqs, H, dk, dv, dt, algo);
    if (st != KDA_OK) return st;
    if (gate != KDA_GATE_LOWER_BOUNDED && gate != KDA_GATE_SOFTPLUS) return KDA_ERR_INVALID_ARG;
    if (checkpoint_every < 0 || checkpoint_every % 64 != 0) return KDA_ERR_INVALID_ARG;
    if (checkpoint_every > 0 && (!checkpoints || !aligned(checkpoints, 16))) return KDA_ERR_INVALID_ARG;
    if (checkpoint_every > 0 && algo == KDA_ALGO_TENSOR_CORE_SPLIT) return KDA_ERR_UNSUPPORTED;
    if (num_seqs > 0 && !cu_seqlens_dev) return KDA_ERR_INVALID_ARG;
    if (total_tokens > 0 && (!q || !k || !v || !z || !A || !beta || !o)) return KDA_ERR_INVALID_ARG;
    for (const void *p : {q, k, v, z, (const void *)o, (const void *)initial_state,
                          (const void *)final_state, (const void *)workspace})
        if (p && !aligned(p, 16)) return KDA_ERR_INVALID_ARG;
    if ((A && !aligned(A, 4)) || (beta && !aligned(beta, 4)) ||
        (cu_seqlens_dev && !aligned(cu_seqlens_dev, 4)))
        return KDA_ERR_INVALID_ARG;
    if (cu_seqlens_host) {
        if (cu_seqlens_host[0] != 0 || cu_seqlens_host[num_seqs] != total_tokens)
            return KDA_ERR_INVALID_ARG;
        for (int32_t i = 0; i < num_seqs; ++i)
            if (cu_seqlens_host[i + 1] < cu_seqlens_host[i]) return KDA_ERR_INVALID_ARG;
    }
    if (num_seqs == 0) return KDA_OK;
    const size_t need = kda_prefill_gated_workspace_size(total_tokens, num_seqs, H, dk, dv, dt,
                                                         algo, gate);
    if (need > 0 && (!workspace || workspace_bytes < need)) return KDA_ERR_WORKSPACE;

    int32_t *status = nullptr;
    if ((st = status_word(&status)) != KDA_OK) return st;

    kda::PrefillArgs a;
    a.q = q; a.k = k; a.v = v; a.z = z; a.A = A; a.beta = beta;
    a.cu_seqlens = cu_seqlens_dev; a.seq_order = nullptr;
    a.num_seqs = num_seqs; a.total_tokens = total_tokens; a.H = H; a.dk = dk; a.dv = dv;
    a.bf16 = (dt == KDA_DTYPE_BF16);
    a.initial_state = initial_state; a.final_state = final_state; a.o = o;
    a.workspace = workspace; a.workspace_bytes = workspace_bytes; a.status = status;
    a.events = stage_events; a.num_events = stage_events ? num_stage_events : 0;
    a.ckpt_every = checkpoint_every; a.checkpoints = checkpoint_every > 0 ? checkpoints : nullptr;
    // Checkpoints come from the unsplit state chain; AUTO then keeps every
    // sequence whole (its workspace, sized for a split, is large enough).
    a.segments = checkpoint_every > 0 ? 1 : segments_for(total_tokens, num_seqs, H, dk, dv, dt, algo);
    a.gate = gate == KDA_GATE_SOFTPLUS ? 1 : 0;
    if (dbg) {
        a.dbg_G = dbg[0]; a.dbg_W = dbg[1]; a.dbg_U = dbg[2]; a.dbg_delta = dbg[3];
    }

    cudaError_t err = use_tensor_core(dk, dv, dt, algo)
                          ? kda::launch_prefill_tensor_core(a, (cudaStream_t)stream)
                          : kda::launch_prefill_cuda_core(a, (cudaStream_t)stream);
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // namespace

extern "C" kda_status kda_prefill_checkpointed(
    const void *q, const void *k, const void *v, const void *z, const float *A, const float *beta,
    const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host, int32_t num_seqs,
    int32_t total_tokens, int32_t H, int32_t dk, int32_t dv, kda_dtype dt,
    const float *initial_state, float *final_state, void *o, void *workspace,
    size_t workspace_bytes, kda_algo algo, void *stream, void *const *stage_events,
    int32_t num_stage_events, int32_t checkpoint_every, float *checkpoints)
{
    return prefill_impl(q, k, v, z, A, beta, cu_seqlens_dev, cu_seqlens_host, num_seqs,
                        total_tokens, H, dk, dv, dt, initial_state, final_state, o, workspace,
                        workspace_bytes, algo, stream, stage_events, num_stage_events,
                        checkpoint_every, checkpoints, KDA_GATE_LOWER_BOUNDED);
}

extern "C" kda_status kda_prefill_debug(const void *q, const void *k, const void *v, const void *z,
                                        const float *A, const float *beta,
                                        const int32_t *cu_seqlens_dev,
                                        const int32_t *cu_seqlens_host, int32_t num_seqs,
                                        int32_t total_tokens, int32_t H, int32_t dk, int32_t dv,
                                        kda_dtype dt, const float *initial_state,
                                        float *final_state, void *o, void *workspace,
                                        size_t workspace_bytes, float *G_out, float *W_out,
                                        float *U_out, float *delta_out, void *stream)
{
    if (dt != KDA_DTYPE_BF16 || dk != 128 || dv != 128) {
        const kda_status st = check_prefill_sizes(total_tokens, num_seqs, H, dk, dv, dt,
                                                  KDA_ALGO_TENSOR_CORE);
        return st != KDA_OK ? st : KDA_ERR_UNSUPPORTED;
    }
    for (const float *p : {(const float *)G_out, (const float *)W_out, (const float *)U_out,
                           (const float *)delta_out})
        if (p && !aligned(p, 16)) return KDA_ERR_INVALID_ARG;
    float *const dbg[4] = {G_out, W_out, U_out, delta_out};
    return prefill_impl(q, k, v, z, A, beta, cu_seqlens_dev, cu_seqlens_host, num_seqs,
                        total_tokens, H, dk, dv, dt, initial_state, final_state, o, workspace,
                        workspace_bytes, KDA_ALGO_TENSOR_CORE, stream, nullptr, 0, 0, nullptr,
                        KDA_GATE_LOWER_BOUNDED, dbg);
}

extern "C" kda_status kda_decode_check_slots(const int32_t *slots_host, int32_t B, int32_t pool_size)
{
    if (B < 0 || pool_size < 0 || (B > 0 && !slots_host)) return KDA_ERR_INVALID_ARG;
    std::vector<uint8_t> seen((size_t)pool_size, 0);
    for (int32_t b = 0; b < B; ++b) {
        const int32_t sl = slots_host[b];
        if (sl < 0 || sl >= pool_size || seen[(size_t)sl]) return KDA_ERR_INVALID_ARG;
        seen[(size_t)sl] = 1;
    }
    return KDA_OK;
}

extern "C" kda_status kda_prefill_gated(const void *q, const void *k, const void *v, const void *z,
                                        const float *A, const float *beta,
                                        const int32_t *cu_seqlens_dev,
                                        const int32_t *cu_seqlens_host, int32_t num_seqs,
                                        int32_t total_tokens, int32_t H, int32_t dk, int32_t dv,
                                        kda_dtype dt, const float *initial_state,
                                        float *final_state, void *o, void *workspace,
                                        size_t workspace_bytes, kda_algo algo, kda_gate gate,
                                        void *stream)
{
    return prefill_impl(q, k, v, z, A, beta, cu_seqlens_dev, cu_seqlens_host, num_seqs,
                        total_tokens, H, dk, dv, dt, initial_state, final_state, o, workspace,
                        workspace_bytes, algo, stream, nullptr, 0, 0, nullptr, gate);
}

extern "C" kda_status kda_prefill_ex(const void *q, const void *k, const void *v, const void *z,
                                     const float *A, const float *beta,
                                     const int32_t *cu_seqlens_dev,
                                     const int32_t *cu_seqlens_host, int32_t num_seqs,
                                     int32_t total_tokens, int32_t H, int32_t dk, int32_t dv,
                                     kda_dtype dt, const float *initial_state,
                                     float *final_state, void *o, void *workspace,
                                     size_t workspace_bytes, kda_algo algo, void *stream,
                                     void *const *stage_events, int32_t num_stage_events)
{
    return kda_prefill_checkpointed(q, k, v, z, A, beta, cu_seqlens_dev, cu_seqlens_host,
                                    num_seqs, total_tokens, H, dk, dv, dt, initial_state,
                                    final_state, o, workspace, workspace_bytes, algo, stream,
                                    stage_events, num_stage_events, 0, nullptr);
}

extern "C" kda_status kda_prefill(const void *q, const void *k, const void *v, const void *z,
                                  const float *A, const float *beta,
                                  const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                                  int32_t num_seqs, int32_t total_tokens, int32_t H, int32_t dk,
                                  int32_t dv, kda_dtype dt, const float *initial_state,
                                  float *final_state, void *o, void *workspace,
                                  size_t workspace_bytes, void *stream)
{
    return kda_prefill_ex(q, k, v, z, A, beta, cu_seqlens_dev, cu_seqlens_host, num_seqs,
                          total_tokens, H, dk, dv, dt, initial_state, final_state, o, workspace,
                          workspace_bytes, KDA_ALGO_AUTO, stream, nullptr, 0);
}

extern "C" int32_t kda_prefill_kernel_count(int32_t total_tokens, int32_t num_seqs, int32_t H,
                                            int32_t dk, int32_t dv, kda_dtype dt, kda_algo algo)
{
    if (check_prefill_sizes(total_tokens, num_seqs, H, dk, dv, dt, algo) != KDA_OK) return 0;
    if (!use_tensor_core(dk, dv, dt, algo)) return 1;
    return segments_for(total_tokens, num_seqs, H, dk, dv, dt, algo) > 1 ? 5 : 3;
}

extern "C" kda_status kda_decode_step(const void *q, const void *k, const void *v, const void *z,
                                      const float *A, const float *beta, int32_t B, int32_t H,
                                      int32_t dk, int32_t dv, kda_dtype dt, float *state,
                                      int32_t pool_size, const int32_t *slots, void *o,
                                      void *stream)
{
    return kda_decode_step_gated(q, k, v, z, A, beta, B, H, dk, dv, dt, state, pool_size, slots, o,
                                 KDA_GATE_LOWER_BOUNDED, stream);
}

extern "C" kda_status kda_decode_step_gated(const void *q, const void *k, const void *v,
                                            const void *z, const float *A, const float *beta,
                                            int32_t B, int32_t H, int32_t dk, int32_t dv,
                                            kda_dtype dt, float *state, int32_t pool_size,
                                            const int32_t *slots, void *o, kda_gate gate,
                                            void *stream)
{
    if (B < 0 || H <= 0 || pool_size < 0) return KDA_ERR_INVALID_ARG;
    if (gate != KDA_GATE_LOWER_BOUNDED && gate != KDA_GATE_SOFTPLUS) return KDA_ERR_INVALID_ARG;
    if (dt != KDA_DTYPE_BF16 && dt != KDA_DTYPE_F32) return KDA_ERR_INVALID_ARG;
    if (dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if (B == 0) return KDA_OK;
    if (!q || !k || !v || !z || !A || !beta || !state || !o) return KDA_ERR_INVALID_ARG;
    if (!slots && pool_size < B) return KDA_ERR_INVALID_ARG;
    for (const void *p : {q, k, v, z, (const void *)o, (const void *)state})
        if (!aligned(p, 16)) return KDA_ERR_INVALID_ARG;
    if (!aligned(A, 4) || !aligned(beta, 4) || (slots && !aligned(slots, 4)))
        return KDA_ERR_INVALID_ARG;

    kda::DecodeArgs a;
    a.q = q; a.k = k; a.v = v; a.z = z; a.A = A; a.beta = beta;
    a.B = B; a.H = H; a.dk = dk; a.dv = dv; a.bf16 = (dt == KDA_DTYPE_BF16);
    a.state = state; a.slots = slots; a.o = o;
    a.gate = gate == KDA_GATE_SOFTPLUS ? 1 : 0;
    cudaError_t err = kda::launch_decode_step(a, (cudaStream_t)stream);
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

extern "C" kda_status kda_decode_multi(const void *q, const void *k, const void *v, const void *z,
                                       const float *A, const float *beta, int32_t B, int32_t Tq,
                                       int32_t H, int32_t dk, int32_t dv, kda_dtype dt,
                                       float *state, int32_t pool_size, const int32_t *slots,
                                       const int32_t *num_tokens, int32_t update_state, void *o,
                                       void *stream)
{
    if (B < 0 || H <= 0 || pool_size < 0 || Tq < 1 || Tq > 64) return KDA_ERR_INVALID_ARG;
    if (dt != KDA_DTYPE_BF16 && dt != KDA_DTYPE_F32) return KDA_ERR_INVALID_ARG;
    if (update_state != 0 && update_state != 1) return KDA_ERR_INVALID_ARG;
    if (dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if (B == 0) return KDA_OK;
    if (!q || !k || !v || !z || !A || !beta || !state) return KDA_ERR_INVALID_ARG;
    if (!o && !update_state) return KDA_ERR_INVALID_ARG;   // verify without outputs does nothing
    if (!slots && pool_size < B) return KDA_ERR_INVALID_ARG;
    for (const void *p : {q, k, v, z, (const void *)o, (const void *)state})
        if (p && !aligned(p, 16)) return KDA_ERR_INVALID_ARG;
    if (!aligned(A, 4) || !aligned(beta, 4) || (slots && !aligned(slots, 4)) ||
        (num_tokens && !aligned(num_tokens, 4)))
        return KDA_ERR_INVALID_ARG;

    int32_t *status = nullptr;
    kda_status st = status_word(&status);
    if (st != KDA_OK) return st;

    kda::DecodeMultiArgs a;
    a.q = q; a.k = k; a.v = v; a.z = z; a.A = A; a.beta = beta;
    a.B = B; a.Tq = Tq; a.H = H; a.dk = dk; a.dv = dv; a.bf16 = (dt == KDA_DTYPE_BF16);
    a.state = state; a.slots = slots; a.num_tokens = num_tokens;
    a.update_state = update_state != 0; a.o = o; a.status = status;
    cudaError_t err = kda::launch_decode_multi(a, (cudaStream_t)stream);
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

extern "C" kda_status kda_device_status(void *stream, int32_t *status_out)
{
    if (!status_out) return KDA_ERR_INVALID_ARG;
    int32_t *word = nullptr;
    kda_status st = status_word(&word);
    if (st != KDA_OK) return st;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return KDA_ERR_CUDA;
    int32_t v = 0, zero = 0;
    if (cudaMemcpy(&v, word, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return KDA_ERR_CUDA;
    if (cudaMemcpy(word, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
        return KDA_ERR_CUDA;
    *status_out = v;
    return KDA_OK;
}

extern "C" kda_status kda_selftest_wait_timeout(int64_t limit_ns, void *stream)
{
    if (limit_ns < 1000000LL || limit_ns > 10000000000LL) return KDA_ERR_INVALID_ARG;
    int32_t *word = nullptr;
    kda_status st = status_word(&word);
    if (st != KDA_OK) return st;
    return kda::launch_wait_timeout_selftest(word, limit_ns, (cudaStream_t)stream) == cudaSuccess
               ? KDA_OK
               : KDA_ERR_CUDA;
}
