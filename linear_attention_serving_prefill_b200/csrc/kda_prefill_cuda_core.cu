// Chunked KDA prefill on CUDA cores, fp32 arithmetic throughout (the check mode).
//
// One CTA owns one (sequence, head, 32-wide slice of dv) and walks the sequence
// in 16-token chunks -- the "secondary tile" of "Kimi K3: Architecture, Training,
// and Million-Token Agentic RL", section 3.3 -- carrying its dk x 32 fp32 state
// slice in shared memory.  Columns of S are independent (v enters column-wise),
// so slices never communicate.  Per chunk, with G the inclusive cumulative
// log-decay inside the chunk (G in [-80, 0] because g >= -5):
//
//   Kt = K*e^{G}, Kh = K*e^{-G}, Qt = Q*e^{G}, Kd = K*e^{G_last - G}
//   A  = strictly_lower(Diag(beta) Kt Kh^T)            (16 x 16)
//   P  = lower_incl_diag(Qt Kh^T)                      (16 x 16)
//   (I + A) D = Diag(beta) (V - Kt S)   -> forward substitution for D
//   O  = Qt S + P D                                    (read after write)
//   S <- Diag(e^{G_last}) S + Kd^T D
//
// which is the recurrence of section 3.1 unrolled over one chunk; the state
// crosses only chunk boundaries (section 3.3 chunk I/O equation).  The e^{-G}
// factor reaches at most e^{80}, finite in fp32 -- the bound section 3.3 gives
// for a 16-token tile.
//
// With the unbounded negative-Softplus gate that section contrasts with the
// bound, e^{-G} overflows and every chunk is a diagonal tile needing the
// position-pair path: A and P take their decays pair by pair,
//   A[r][s] = beta_r sum_c k_rc k_sc e^{G_rc - G_sc},   P[r][s] = sum_c q_rc k_sc e^{G_rc - G_sc},
// each exponent <= 0, and nothing else uses a reciprocal decay.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {
namespace {

constexpr int kC = 16;      // chunk length
constexpr int kDVS = 32;    // dv slice per CTA
constexpr int kThreads = 256;

template <int DK, int GATE>
struct CudaCoreSmem {
    static constexpr int LD = DK + 1;  // padded row stride: conflict-free column walks
    // the pair path keeps the raw q and the cumulative log-decay G besides
    static constexpr int kPair = GATE == kGateSoftplus ? 2 * kC * LD : 0;
    static constexpr int kFloats = 4 * kC * LD + DK * kDVS + 2 * kC * kDVS +
                                   2 * kC * (kC + 1) + 3 * DK + kC + kPair;
    static constexpr size_t kBytes = sizeof(float) * kFloats;
};

template <int DK, typename TIn, int GATE>
__global__ void __launch_bounds__(kThreads)
prefill_cuda_core_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k,
                         const TIn *__restrict__ v, const TIn *__restrict__ z,
                         const float *__restrict__ A, const float *__restrict__ beta,
                         const int32_t *__restrict__ cu_seqlens, int H, int dv,
                         const float *S0, float *Sf, TIn *__restrict__ o, int ckpt_every,
                         float *__restrict__ ckpts)
{
    constexpr int LD = CudaCoreSmem<DK, GATE>::LD;
    constexpr bool kPairPath = GATE == kGateSoftplus;
    extern __shared__ float sm[];
    float *sKt = sm;                  // [kC][LD]  K e^{G}
    float *sKh = sKt + kC * LD;       // [kC][LD]  K e^{-G}
    float *sQt = sKh + kC * LD;       // [kC][LD]  Q e^{G}
    float *sKd = sQt + kC * LD;       // [kC][LD]  g, then G, then K e^{G_last - G}
    float *sS = sKd + kC * LD;        // [DK][kDVS] state slice
    float *sV = sS + DK * kDVS;       // [kC][kDVS] v, then the rhs, then D
    float *sO = sV + kC * kDVS;       // [kC][kDVS] Qt S
    float *sA = sO + kC * kDVS;       // [kC][kC+1]
    float *sP = sA + kC * (kC + 1);   // [kC][kC+1]
    float *sEA = sP + kC * (kC + 1);  // [DK] exp(A[h])
    float *sGL = sEA + DK;            // [DK] G at the chunk's last row
    float *sEGL = sGL + DK;           // [DK] exp(G_last)
    float *sB = sEGL + DK;            // [kC] beta
    float *sQr = sB + kC;             // [kC][LD] raw q   (pair path only)
    float *sG = sQr + kC * LD;        // [kC][LD] G       (pair path only)

    const int nslices = dv / kDVS;
    const int slice = blockIdx.x % nslices;
    const int h = (blockIdx.x / nslices) % H;
    const int n = blockIdx.x / (nslices * H);
    const int j0 = slice * kDVS;
    const int tid = threadIdx.x;
    const int t_begin = cu_seqlens[n], t_end = cu_seqlens[n + 1];
    const size_t state_base = ((size_t)n * H + h) * DK * dv + j0;
    // Row of this sequence's first checkpoint: sum over earlier sequences of L / every.
    __shared__ long long sCkBase;
    if (tid == 0) {
        long long b = 0;
        if (ckpt_every > 0)
            for (int m = 0; m < n; ++m) b += (cu_seqlens[m + 1] - cu_seqlens[m]) / ckpt_every;
        sCkBase = b;
    }

    for (int c = tid; c < DK; c += kThreads) sEA[c] = expf(A[(size_t)h * DK + c]);
    for (int e = tid; e < DK * kDVS; e += kThreads) {
        const int c = e / kDVS, j = e % kDVS;
        sS[e] = S0 ? S0[state_base + (size_t)c * dv + j] : 0.0f;
    }
    __syncthreads();

    for (int tc = t_begin; tc < t_end; tc += kC) {
        const int len = min(kC, t_end - tc);
        // Load the chunk; rows past the sequence end are zero (k = q = v = 0,
        // beta = 0, g = 0), which leaves the state and every valid row unchanged.
        for (int e = tid; e < kC * DK; e += kThreads) {
            const int r = e / DK, c = e % DK;
            float kv = 0.f, qv = 0.f, gv = 0.f;
            if (r < len) {
                const size_t idx = ((size_t)(tc + r) * H + h) * DK + c;
                kv = to_f32(k[idx]);
                qv = to_f32(q[idx]);
                gv = gate_fn<GATE>(sEA[c], to_f32(z[idx]));
            }
            sKt[r * LD + c] = kv;
            sQt[r * LD + c] = qv;
            sKd[r * LD + c] = gv;
        }
        for (int e = tid; e < kC * kDVS; e += kThreads) {
            const int r = e / kDVS, j = e % kDVS;
            sV[e] = r < len ? to_f32(v[((size_t)(tc + r) * H + h) * dv + j0 + j]) : 0.f;
        }
        if (tid < kC) sB[tid] = tid < len ? beta[(size_t)(tc + tid) * H + h] : 0.f;
        __syncthreads();

        // Inclusive cumulative log-decay per key channel.
        for (int c = tid; c < DK; c += kThreads) {
            float acc = 0.f;
            for (int r = 0; r < kC; ++r) {
                acc += sKd[r * LD + c];
                sKd[r * LD + c] = acc;
            }
            sGL[c] = acc;
            sEGL[c] = expf(acc);
        }
        __syncthreads();

        for (int e = tid; e < kC * DK; e += kThreads) {
            const int r = e / DK, c = e % DK;
            const float G = sKd[r * LD + c], kv = sKt[r * LD + c], qv = sQt[r * LD + c];
            const float eg = expf(G);
            sKt[r * LD + c] = kv * eg;
            sQt[r * LD + c] = qv * eg;
            sKd[r * LD + c] = kv * expf(sGL[c] - G);
            if (kPairPath) {
                sKh[r * LD + c] = kv;   // raw k, q and G for the pair decays
                sQr[r * LD + c] = qv;
                sG[r * LD + c] = G;
            } else {
                sKh[r * LD + c] = kv * expf(-G);
            }
        }
        __syncthreads();

        // A and P: one (r, s) pair per thread.
        {
            const int r = tid / kC, s = tid % kC;
            float a = 0.f, p = 0.f;
            if (kPairPath) {
                if (s <= r) {
#pragma unroll 4
                    for (int c = 0; c < DK; ++c) {
                        const float e = expf(sG[r * LD + c] - sG[s * LD + c]);  // <= 1
                        const float ke = sKh[s * LD + c] * e;
                        a = fmaf(sKh[r * LD + c], ke, a);
                        p = fmaf(sQr[r * LD + c], ke, p);
                    }
                }
            } else {
#pragma unroll 8
                for (int c = 0; c < DK; ++c) {
                    const float kh = sKh[s * LD + c];
                    a = fmaf(sKt[r * LD + c], kh, a);
                    p = fmaf(sQt[r * LD + c], kh, p);
                }
            }
            sA[r * (kC + 1) + s] = s < r ? sB[r] * a : 0.f;
            sP[r * (kC + 1) + s] = s <= r ? p : 0.f;
        }
        // rhs = Diag(beta)(V - Kt S) and O1 = Qt S: rows r0 and r0 + 8, column j.
        {
            const int j = tid % kDVS, r0 = tid / kDVS;
            float k0 = 0.f, k1 = 0.f, q0 = 0.f, q1 = 0.f;
#pragma unroll 8
            for (int c = 0; c < DK; ++c) {
                const float s = sS[c * kDVS + j];
                k0 = fmaf(sKt[r0 * LD + c], s, k0);
                k1 = fmaf(sKt[(r0 + 8) * LD + c], s, k1);
                q0 = fmaf(sQt[r0 * LD + c], s, q0);
                q1 = fmaf(sQt[(r0 + 8) * LD + c], s, q1);
            }
            sV[r0 * kDVS + j] = sB[r0] * (sV[r0 * kDVS + j] - k0);
            sV[(r0 + 8) * kDVS + j] = sB[r0 + 8] * (sV[(r0 + 8) * kDVS + j] - k1);
            sO[r0 * kDVS + j] = q0;
            sO[(r0 + 8) * kDVS + j] = q1;
        }
        __syncthreads();

        // (I + A) D = rhs by forward substitution, one column per thread.
        if (tid < kDVS) {
            const int j = tid;
            for (int r = 1; r < kC; ++r) {
                float acc = sV[r * kDVS + j];
                for (int s = 0; s < r; ++s) acc = fmaf(-sA[r * (kC + 1) + s], sV[s * kDVS + j], acc);
                sV[r * kDVS + j] = acc;
            }
        }
        __syncthreads();

        // O = Qt S + P D for the valid rows.
        {
            const int j = tid % kDVS, r0 = tid / kDVS;
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int r = r0 + 8 * rr;
                float acc = sO[r * kDVS + j];
                for (int s = 0; s <= r; ++s) acc = fmaf(sP[r * (kC + 1) + s], sV[s * kDVS + j], acc);
                if (r < len) o[((size_t)(tc + r) * H + h) * dv + j0 + j] = from_f32<TIn>(acc);
            }
        }
        // S <- Diag(e^{G_last}) S + Kd^T D.
        {
            const int j = tid % kDVS;
            for (int c = tid / kDVS; c < DK; c += kThreads / kDVS) {
                float acc = sEGL[c] * sS[c * kDVS + j];
#pragma unroll
                for (int r = 0; r < kC; ++r) acc = fmaf(sKd[r * LD + c], sV[r * kDVS + j], acc);
                sS[c * kDVS + j] = acc;
            }
        }
        __syncthreads();
        // Checkpoint: the state after the first `pos` tokens, when pos is a multiple of every.
        const int pos = tc + len - t_begin;
        if (ckpt_every > 0 && pos % ckpt_every == 0) {
            const size_t row = (size_t)(sCkBase + pos / ckpt_every - 1);
            for (int e = tid; e < DK * kDVS; e += kThreads) {
                const int c = e / kDVS, j = e % kDVS;
                ckpts[(row * H + h) * DK * dv + (size_t)c * dv + j0 + j] = sS[e];
            }
        }
    }

    if (Sf) {
        for (int e = tid; e < DK * kDVS; e += kThreads) {
            const int c = e / kDVS, j = e % kDVS;
            Sf[state_base + (size_t)c * dv + j] = sS[e];
        }
    }
}

template <int DK, typename TIn, int GATE>
cudaError_t launch_gated(const PrefillArgs &a, cudaStream_t stream)
{
    const size_t smem = CudaCoreSmem<DK, GATE>::kBytes;
    auto kern = prefill_cuda_core_kernel<DK, TIn, GATE>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
    if (err != cudaSuccess) return err;
    const long long blocks = (long long)a.num_seqs * a.H * (a.dv / kDVS);
    if (blocks == 0) return cudaSuccess;
    a.mark(0, stream);
    kern<<<(unsigned)blocks, kThreads, smem, stream>>>(
        (const TIn *)a.q, (const TIn *)a.k, (const TIn *)a.v, (const TIn *)a.z, a.A, a.beta,
        a.cu_seqlens, a.H, a.dv, a.initial_state, a.final_state, (TIn *)a.o, a.ckpt_every,
        a.checkpoints);
    a.mark(1, stream);
    return cudaGetLastError();
}

template <int DK, typename TIn>
cudaError_t launch_typed(const PrefillArgs &a, cudaStream_t stream)
{
    return a.gate == kGateSoftplus ? launch_gated<DK, TIn, kGateSoftplus>(a, stream)
                                   : launch_gated<DK, TIn, kGateBounded>(a, stream);
}

}  // namespace

cudaError_t launch_prefill_cuda_core(const PrefillArgs &a, cudaStream_t stream)
{
    switch (a.dk) {
    case 32: return a.bf16 ? launch_typed<32, __nv_bfloat16>(a, stream) : launch_typed<32, float>(a, stream);
    case 64: return a.bf16 ? launch_typed<64, __nv_bfloat16>(a, stream) : launch_typed<64, float>(a, stream);
    case 128: return a.bf16 ? launch_typed<128, __nv_bfloat16>(a, stream) : launch_typed<128, float>(a, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace kda
