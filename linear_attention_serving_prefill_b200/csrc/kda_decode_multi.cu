// Multi-token decode for speculative decoding: verify and replay.
//
// "Kimi K3 Under the Hood", section "Serving two incompatible cache types":
// rejected draft tokens must not advance the recurrent state, and saving a state
// per draft position would multiply memory traffic, so the projected inputs of
// the drafts are kept and the accepted tokens are replayed on-chip in one fused
// recurrence.  This kernel runs Tq tokens of one (sequence, head) against a state
// read from HBM once and held in registers, in the section 3.2 edit order per
// token (Sbar = Diag(alpha) S; vhat = Sbar^T k; p = Sbar^T q; d = beta (v - vhat);
// S = Sbar + k d^T; o = p + (k . q) d):
//   * verify (update_state = 0): o for every draft token; the state in HBM is
//     not written, so a rejected draft leaves no trace;
//   * replay (update_state = 1): the first num_tokens[b] tokens advance the state,
//     which is written back in place once.
// One CTA of 256 threads per (sequence, head); thread (rg, cg) holds rows
// rg, rg + RG, ... of float4 column group cg, as in the single-token kernel.
// The inputs of kGroup tokens at a time are fetched together into shared
// memory (one memory latency per group, not one per token) before the group's
// sequential token steps run on the register-resident state.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kGroup = 8;   // tokens whose inputs are fetched together

template <int DK, int DV, typename TIn>
__global__ void __launch_bounds__(kThreads)
decode_multi_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k,
                    const TIn *__restrict__ v, const TIn *__restrict__ z,
                    const float *__restrict__ A, const float *__restrict__ beta, int Tq, int H,
                    float *__restrict__ state, const int32_t *__restrict__ slots,
                    const int32_t *__restrict__ num_tokens, int update_state,
                    TIn *__restrict__ o)
{
    constexpr int CG = DV / 4;
    constexpr int RG = kThreads / CG;
    constexpr int RPT = DK / RG;
    static_assert(RPT >= 1 && RG * CG == kThreads, "bad decode tiling");

    __shared__ float sEA[DK];
    __shared__ float sAlphaG[kGroup][DK], sKG[kGroup][DK], sQG[kGroup][DK], sVG[kGroup][DV];
    __shared__ float sBetaG[kGroup];
    __shared__ float4 sRedV[RG][CG], sRedP[RG][CG];
    __shared__ float4 sDelta[CG];
    __shared__ float sKQ;

    const int bh = blockIdx.x;
    const int b = bh / H, h = bh % H;
    const int slot = slots ? slots[b] : b;
    int n_tok = num_tokens ? num_tokens[b] : Tq;
    n_tok = n_tok < 0 ? 0 : (n_tok > Tq ? Tq : n_tok);
    const int tid = threadIdx.x;
    const int cg = tid % CG, rg = tid / CG;
    float4 *S4 = reinterpret_cast<float4 *>(state + ((size_t)slot * H + h) * DK * DV);

    float4 s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) s[i] = S4[(size_t)(rg + i * RG) * CG + cg];
    for (int c = tid; c < DK; c += kThreads) sEA[c] = expf(A[(size_t)h * DK + c]);

    for (int t = 0; t < n_tok; ++t) {
        const int tg = t % kGroup;
        const size_t tok = ((size_t)b * Tq + t) * H + h;   // [B, Tq, H, ...]
        __syncthreads();  // the previous token's reads of the group buffers and sDelta are done
        if (tg == 0) {
            // Inputs of tokens t .. t + kGroup - 1 (those that exist), all loads in flight together.
            const int ng = min(kGroup, n_tok - t);
            for (int e = tid; e < ng * DK; e += kThreads) {
                const int u = e / DK, c = e % DK;
                const size_t tu = ((size_t)b * Tq + t + u) * H + h;
                sAlphaG[u][c] = expf(gate_log_decay(sEA[c], to_f32(z[tu * DK + c])));
                sKG[u][c] = to_f32(k[tu * DK + c]);
                sQG[u][c] = to_f32(q[tu * DK + c]);
            }
            for (int e = tid; e < ng * DV; e += kThreads) {
                const int u = e / DV, jv = e % DV;
                sVG[u][jv] = to_f32(v[(((size_t)b * Tq + t + u) * H + h) * DV + jv]);
            }
            if (tid < ng) sBetaG[tid] = beta[((size_t)b * Tq + t + tid) * H + h];
            __syncthreads();
        }
        const float *sAlpha = sAlphaG[tg], *sK = sKG[tg], *sQ = sQG[tg];
        if (tid < 32) {
            float acc = 0.f;
            for (int c = tid; c < DK; c += 32) acc = fmaf(sK[c], sQ[c], acc);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (tid == 0) sKQ = acc;
        }
        float4 vh = make_float4(0.f, 0.f, 0.f, 0.f), p = vh;
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const int c = rg + i * RG;
            const float a = sAlpha[c], kc = sK[c], qc = sQ[c];
            s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
            vh.x = fmaf(kc, s[i].x, vh.x); vh.y = fmaf(kc, s[i].y, vh.y);
            vh.z = fmaf(kc, s[i].z, vh.z); vh.w = fmaf(kc, s[i].w, vh.w);
            p.x = fmaf(qc, s[i].x, p.x); p.y = fmaf(qc, s[i].y, p.y);
            p.z = fmaf(qc, s[i].z, p.z); p.w = fmaf(qc, s[i].w, p.w);
        }
        sRedV[rg][cg] = vh;
        sRedP[rg][cg] = p;
        __syncthreads();
        if (tid < CG) {
            float4 tv = sRedV[0][tid], tp = sRedP[0][tid];
            for (int r = 1; r < RG; ++r) {
                const float4 a = sRedV[r][tid], c = sRedP[r][tid];
                tv.x += a.x; tv.y += a.y; tv.z += a.z; tv.w += a.w;
                tp.x += c.x; tp.y += c.y; tp.z += c.z; tp.w += c.w;
            }
            const float bt = sBetaG[tg];
            const size_t vo = tok * DV + (size_t)tid * 4;
            const float4 vv = *(const float4 *)&sVG[tg][4 * tid];
            float4 d;
            d.x = bt * (vv.x - tv.x);
            d.y = bt * (vv.y - tv.y);
            d.z = bt * (vv.z - tv.z);
            d.w = bt * (vv.w - tv.w);
            sDelta[tid] = d;
            if (o) {
                const float kq = sKQ;
                o[vo + 0] = from_f32<TIn>(fmaf(kq, d.x, tp.x));
                o[vo + 1] = from_f32<TIn>(fmaf(kq, d.y, tp.y));
                o[vo + 2] = from_f32<TIn>(fmaf(kq, d.z, tp.z));
                o[vo + 3] = from_f32<TIn>(fmaf(kq, d.w, tp.w));
            }
        }
        __syncthreads();
        const float4 d = sDelta[cg];
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const float kc = sK[rg + i * RG];
            s[i].x = fmaf(kc, d.x, s[i].x); s[i].y = fmaf(kc, d.y, s[i].y);
            s[i].z = fmaf(kc, d.z, s[i].z); s[i].w = fmaf(kc, d.w, s[i].w);
        }
    }
    if (update_state && n_tok > 0) {
#pragma unroll
        for (int i = 0; i < RPT; ++i) S4[(size_t)(rg + i * RG) * CG + cg] = s[i];
    }
}

template <int DK, int DV, typename TIn>
cudaError_t launch_typed(const DecodeMultiArgs &a, cudaStream_t stream)
{
    const long long blocks = (long long)a.B * a.H;
    if (blocks == 0) return cudaSuccess;
    decode_multi_kernel<DK, DV, TIn><<<(unsigned)blocks, kThreads, 0, stream>>>(
        (const TIn *)a.q, (const TIn *)a.k, (const TIn *)a.v, (const TIn *)a.z, a.A, a.beta,
        a.Tq, a.H, a.state, a.slots, a.num_tokens, a.update_state ? 1 : 0, (TIn *)a.o);
    return cudaGetLastError();
}

template <int DK, typename TIn>
cudaError_t launch_dv(const DecodeMultiArgs &a, cudaStream_t stream)
{
    switch (a.dv) {
    case 32: return launch_typed<DK, 32, TIn>(a, stream);
    case 64: return launch_typed<DK, 64, TIn>(a, stream);
    case 128: return launch_typed<DK, 128, TIn>(a, stream);
    default: return cudaErrorInvalidValue;
    }
}

template <typename TIn>
cudaError_t launch_dk(const DecodeMultiArgs &a, cudaStream_t stream)
{
    switch (a.dk) {
    case 32: return launch_dv<32, TIn>(a, stream);
    case 64: return launch_dv<64, TIn>(a, stream);
    case 128: return launch_dv<128, TIn>(a, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_decode_multi(const DecodeMultiArgs &a, cudaStream_t stream)
{
    return a.bf16 ? launch_dk<__nv_bfloat16>(a, stream) : launch_dk<float>(a, stream);
}

}  // namespace kda
