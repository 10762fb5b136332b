// kda_prefill_noalloc: the tensor-core prefill with its scratch memory in a
// fixed, file-scope device array instead of a caller-provided workspace.
//
// Some callers cannot allocate device memory when they call the mixer: a
// serving engine that hands all free HBM to its paged cache pool at start-up
// and forbids later allocations, code that runs under another framework's
// allocator with no way to reach it, or a latency-critical loop that cannot
// afford the implicit device synchronisation of cudaMalloc / cudaFree.  This
// entry point needs no workspace from them: the scratch lives in the array
// below, which every GPU that loads this module holds until the process exits.
#include <mutex>
#include <stdint.h>

#include "kda.h"
#include "kda_internal.h"

namespace {

// Largest scratch a call may need: 64 MiB, i.e. about 900 (64-token chunk,
// head) tiles -- for example one 576-token sequence at 96 heads.
constexpr size_t kNoAllocScratchBytes = 64ull << 20;

}  // namespace

// The scratch itself.  Host code must not pass `g_kda_noalloc_scratch` to a
// kernel: on the host that name is only a stand-in for the symbol, not a
// device address.  The device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_kda_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {nullptr};
unsigned long long g_scratch_ctx[kMaxDevices] = {0};

// Device address of the scratch array on the current device, looked up once
// per device and context (the first call on each device does this set-up; it
// is also where the runtime, which loads device code lazily, first places the
// array in that device's memory).  A device reset destroys the context, and
// the module with it; the next call sees a new context id and looks again.
kda_status scratch_on_current_device(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KDA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    unsigned long long ctx = 0;
    const bool have_ctx = kda::current_context_id(&ctx);
    if (!g_scratch_ptr[dev] || !have_ctx || ctx != g_scratch_ctx[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_kda_noalloc_scratch) != cudaSuccess || !p) return KDA_ERR_CUDA;
        g_scratch_ptr[dev] = p;
        g_scratch_ctx[dev] = kda::current_context_id(&ctx) ? ctx : 0;
    }
    *out = g_scratch_ptr[dev];
    return KDA_OK;
}

}  // namespace

extern "C" kda_status kda_prefill_noalloc(const void *q, const void *k, const void *v,
                                          const void *z, const float *A, const float *beta,
                                          const int32_t *cu_seqlens_dev,
                                          const int32_t *cu_seqlens_host, int32_t num_seqs,
                                          int32_t total_tokens, int32_t H, int32_t dk, int32_t dv,
                                          kda_dtype dt, const float *initial_state,
                                          float *final_state, void *o, void *stream)
{
    const size_t need = kda_prefill_workspace_size(total_tokens, num_seqs, H, dk, dv, dt,
                                                   KDA_ALGO_TENSOR_CORE);
    if (need > kNoAllocScratchBytes) return KDA_ERR_WORKSPACE;
    void *scratch = nullptr;
    if (need > 0) {
        const kda_status st = scratch_on_current_device(&scratch);
        if (st != KDA_OK) return st;
    }
    // Invalid arguments (need == 0 for them) are reported by kda_prefill_ex.
    return kda_prefill_ex(q, k, v, z, A, beta, cu_seqlens_dev, cu_seqlens_host, num_seqs,
                          total_tokens, H, dk, dv, dt, initial_state, final_state, o, scratch,
                          kNoAllocScratchBytes, KDA_ALGO_TENSOR_CORE, stream, nullptr, 0);
}
