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
// One CTA of 2 dv threads per (sequence, head).  Warp w owns the 16 value
// columns 16 w .. 16 w + 15 (four float4 column groups) for all dk rows: lane
// (rg, c4) = (lane / 4, lane % 4) holds rows rg, rg + 8, ... of column group
// 4 w + c4 in registers.  Columns of S never mix, so every reduction of a token
// step (vhat and p over the key channels) stays inside a warp (three xor
// shuffles over the row groups), and the token steps need no block barrier:
// each warp runs its own columns' recurrence.  The inputs of kGroup tokens at
// a time, their decays and k.q, are fetched together into shared memory (one
// memory latency and two barriers per group, not per token).
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {
namespace {

constexpr int kGroup = 8;   // tokens whose inputs are fetched together

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) { return __fmul2_rn(a, b); }

template <int DK, int DV, typename TIn>
__global__ void __launch_bounds__(2 * DV)
decode_multi_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k,
                    const TIn *__restrict__ v, const TIn *__restrict__ z,
                    const float *__restrict__ A, const float *__restrict__ beta, int Tq, int H,
                    float *__restrict__ state, const int32_t *__restrict__ slots,
                    const int32_t *__restrict__ num_tokens, int update_state,
                    TIn *__restrict__ o)
{
    constexpr int CG = DV / 4;        // float4 column groups
    constexpr int NT = 2 * DV;        // 8 row groups x CG column groups
    constexpr int NW = NT / 32;
    constexpr int RPT = DK / 8;       // state rows per thread
    static_assert(CG % 4 == 0 && RPT >= 1, "bad decode tiling");

    __shared__ float sEA[DK];
    __shared__ float sAlphaG[kGroup][DK], sKG[kGroup][DK], sQG[kGroup][DK];
    __shared__ __align__(16) float sVG[kGroup][DV];
    __shared__ float sBetaG[kGroup], sKQG[kGroup];

    const int bh = blockIdx.x;
    const int b = bh / H, h = bh % H;
    const int slot = slots ? slots[b] : b;
    int n_tok = num_tokens ? num_tokens[b] : Tq;
    n_tok = n_tok < 0 ? 0 : (n_tok > Tq ? Tq : n_tok);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rg = lane >> 2, cg = 4 * warp + (lane & 3);
    float4 *S4 = reinterpret_cast<float4 *>(state + ((size_t)slot * H + h) * DK * DV);

    float4 s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) s[i] = S4[(size_t)(rg + 8 * i) * CG + cg];
    for (int c = tid; c < DK; c += NT) sEA[c] = expf(A[(size_t)h * DK + c]);

    for (int t = 0; t < n_tok; ++t) {
        const int tg = t % kGroup;
        if (tg == 0) {
            // Inputs of tokens t .. t + kGroup - 1 (those that exist), all loads in
            // flight together; the previous group's buffers are no longer read.
            __syncthreads();
            const int ng = min(kGroup, n_tok - t);
            for (int e = tid; e < ng * DK; e += NT) {
                const int u = e / DK, c = e % DK;
                const size_t tu = ((size_t)b * Tq + t + u) * H + h;
                sAlphaG[u][c] = expf(gate_log_decay(sEA[c], to_f32(z[tu * DK + c])));
                sKG[u][c] = to_f32(k[tu * DK + c]);
                sQG[u][c] = to_f32(q[tu * DK + c]);
            }
            for (int e = tid; e < ng * DV; e += NT) {
                const int u = e / DV, jv = e % DV;
                sVG[u][jv] = to_f32(v[(((size_t)b * Tq + t + u) * H + h) * DV + jv]);
            }
            if (tid < ng) sBetaG[tid] = beta[((size_t)b * Tq + t + tid) * H + h];
            __syncthreads();
            for (int u = warp; u < ng; u += NW) {     // k . q of each token, one warp each
                float acc = 0.f;
                for (int c = lane; c < DK; c += 32) acc = fmaf(sKG[u][c], sQG[u][c], acc);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
                if (lane == 0) sKQG[u] = acc;
            }
            __syncthreads();
        }
        const float *sAlpha = sAlphaG[tg], *sK = sKG[tg], *sQ = sQG[tg];
        // Sbar = Diag(alpha) S; partial vhat = Sbar^T k and p = Sbar^T q over this
        // thread's rows, as (x, y) and (z, w) pairs.
        float2 vh0 = make_float2(0.f, 0.f), vh1 = vh0, p0 = vh0, p1 = vh0;
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const int c = rg + 8 * i;
            const float a = sAlpha[c], kc = sK[c], qc = sQ[c];
            float2 lo = fmul2(make_float2(s[i].x, s[i].y), make_float2(a, a));
            float2 hi = fmul2(make_float2(s[i].z, s[i].w), make_float2(a, a));
            s[i] = make_float4(lo.x, lo.y, hi.x, hi.y);
            vh0 = ffma2(make_float2(kc, kc), lo, vh0);
            vh1 = ffma2(make_float2(kc, kc), hi, vh1);
            p0 = ffma2(make_float2(qc, qc), lo, p0);
            p1 = ffma2(make_float2(qc, qc), hi, p1);
        }
        // Sum over the 8 row groups (lanes 4 apart).
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            vh0.x += __shfl_xor_sync(0xffffffffu, vh0.x, off);
            vh0.y += __shfl_xor_sync(0xffffffffu, vh0.y, off);
            vh1.x += __shfl_xor_sync(0xffffffffu, vh1.x, off);
            vh1.y += __shfl_xor_sync(0xffffffffu, vh1.y, off);
            p0.x += __shfl_xor_sync(0xffffffffu, p0.x, off);
            p0.y += __shfl_xor_sync(0xffffffffu, p0.y, off);
            p1.x += __shfl_xor_sync(0xffffffffu, p1.x, off);
            p1.y += __shfl_xor_sync(0xffffffffu, p1.y, off);
        }
        // delta = beta (v - vhat); o = p + (k . q) delta; S = Sbar + k delta^T.
        const float bt = sBetaG[tg];
        const float4 vv = *(const float4 *)&sVG[tg][4 * cg];
        const float4 d = make_float4(bt * (vv.x - vh0.x), bt * (vv.y - vh0.y),
                                     bt * (vv.z - vh1.x), bt * (vv.w - vh1.y));
        if (o && rg == 0) {
            const float kq = sKQG[tg];
            const size_t vo = (((size_t)b * Tq + t) * H + h) * DV + (size_t)cg * 4;
            o[vo + 0] = from_f32<TIn>(fmaf(kq, d.x, p0.x));
            o[vo + 1] = from_f32<TIn>(fmaf(kq, d.y, p0.y));
            o[vo + 2] = from_f32<TIn>(fmaf(kq, d.z, p1.x));
            o[vo + 3] = from_f32<TIn>(fmaf(kq, d.w, p1.y));
        }
        const float2 dlo = make_float2(d.x, d.y), dhi = make_float2(d.z, d.w);
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const float kc = sK[rg + 8 * i];
            const float2 lo = ffma2(make_float2(kc, kc), dlo, make_float2(s[i].x, s[i].y));
            const float2 hi = ffma2(make_float2(kc, kc), dhi, make_float2(s[i].z, s[i].w));
            s[i] = make_float4(lo.x, lo.y, hi.x, hi.y);
        }
    }
    if (update_state && n_tok > 0) {
#pragma unroll
        for (int i = 0; i < RPT; ++i) S4[(size_t)(rg + 8 * i) * CG + cg] = s[i];
    }
}

template <int DK, int DV, typename TIn>
cudaError_t launch_typed(const DecodeMultiArgs &a, cudaStream_t stream)
{
    const long long blocks = (long long)a.B * a.H;
    if (blocks == 0) return cudaSuccess;
    decode_multi_kernel<DK, DV, TIn><<<(unsigned)blocks, 2 * DV, 0, stream>>>(
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
