// Single-token KDA decode step ("Kimi K3: Architecture, Training, and
// Million-Token Agentic RL", section 3.2 edit order):
//
//   Sbar = Diag(alpha) S;  vhat = Sbar^T k;  p = Sbar^T q;
//   d = beta (v - vhat);   S <- Sbar + k d^T;  o = S^T q = p + (k . q) d
//
// The last identity lets one pass read S and one pass write it: the state is
// read from HBM once into registers (128-bit loads, dv contiguous), both dk
// reductions run on the decayed copy, and the updated state is written back
// once.  That is the minimum traffic, 2 * dk * dv * 4 bytes per (sequence,
// head), so the kernel is bound by HBM bandwidth.  One CTA of 256 threads owns
// one (sequence, head); thread (rg, cg) holds rows rg, rg + RG, ... of float4
// column group cg, so that every warp reads whole 512-byte rows of the state.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {
namespace {

constexpr int kThreads = 256;

template <int DK, int DV, typename TIn, int GATE>
__global__ void __launch_bounds__(kThreads)
decode_step_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k,
                   const TIn *__restrict__ v, const TIn *__restrict__ z,
                   const float *__restrict__ A, const float *__restrict__ beta, int H,
                   float *__restrict__ state, const int32_t *__restrict__ slots,
                   TIn *__restrict__ o)
{
    constexpr int CG = DV / 4;           // float4 column groups
    constexpr int RG = kThreads / CG;    // row groups
    constexpr int RPT = DK / RG;         // rows per thread
    static_assert(RPT >= 1 && RG * CG == kThreads, "bad decode tiling");

    __shared__ float sAlpha[DK], sK[DK], sQ[DK];
    __shared__ float4 sRedV[RG][CG], sRedP[RG][CG];
    __shared__ float4 sDelta[CG];
    __shared__ float sKQ;

    const int bh = blockIdx.x;
    const int b = bh / H, h = bh % H;
    const int slot = slots ? slots[b] : b;
    const int tid = threadIdx.x;
    const int cg = tid % CG, rg = tid / CG;
    float4 *S4 = reinterpret_cast<float4 *>(state + ((size_t)slot * H + h) * DK * DV);

    // Issue every state load first; the gate math below overlaps their latency.
    float4 s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) s[i] = S4[(size_t)(rg + i * RG) * CG + cg];

    const size_t tok = (size_t)b * H + h;
    if (tid < DK) {
        const float kc = to_f32(k[tok * DK + tid]);
        const float qc = to_f32(q[tok * DK + tid]);
        const float g = gate_fn<GATE>(expf(A[(size_t)h * DK + tid]), to_f32(z[tok * DK + tid]));
        sAlpha[tid] = expf(g);
        sK[tid] = kc;
        sQ[tid] = qc;
    }
    __syncthreads();
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
        // Sum of the RG row-group partials as a pairwise tree, ((0+1)+(2+3))+...,
        // the order of the multi-token kernel's xor butterfly over its 8 row
        // groups: at dv = 128 (RG = 8, rows rg + 8 i in both kernels) a one-token
        // replay there equals this step bit for bit.
        float4 tv, tp;
        {
            float4 v[RG], pp[RG];
#pragma unroll
            for (int r = 0; r < RG; ++r) { v[r] = sRedV[r][tid]; pp[r] = sRedP[r][tid]; }
#pragma unroll
            for (int w = 1; w < RG; w <<= 1)
#pragma unroll
                for (int r = 0; r + w < RG; r += 2 * w) {
                    v[r].x += v[r + w].x; v[r].y += v[r + w].y; v[r].z += v[r + w].z; v[r].w += v[r + w].w;
                    pp[r].x += pp[r + w].x; pp[r].y += pp[r + w].y; pp[r].z += pp[r + w].z; pp[r].w += pp[r + w].w;
                }
            tv = v[0];
            tp = pp[0];
        }
        const float bt = beta[tok];
        const size_t vo = tok * DV + (size_t)tid * 4;
        float4 d;
        d.x = bt * (to_f32(v[vo + 0]) - tv.x);
        d.y = bt * (to_f32(v[vo + 1]) - tv.y);
        d.z = bt * (to_f32(v[vo + 2]) - tv.z);
        d.w = bt * (to_f32(v[vo + 3]) - tv.w);
        sDelta[tid] = d;
        const float kq = sKQ;
        o[vo + 0] = from_f32<TIn>(fmaf(kq, d.x, tp.x));
        o[vo + 1] = from_f32<TIn>(fmaf(kq, d.y, tp.y));
        o[vo + 2] = from_f32<TIn>(fmaf(kq, d.z, tp.z));
        o[vo + 3] = from_f32<TIn>(fmaf(kq, d.w, tp.w));
    }
    __syncthreads();

    const float4 d = sDelta[cg];
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int c = rg + i * RG;
        const float kc = sK[c];
        float4 r;
        r.x = fmaf(kc, d.x, s[i].x); r.y = fmaf(kc, d.y, s[i].y);
        r.z = fmaf(kc, d.z, s[i].z); r.w = fmaf(kc, d.w, s[i].w);
        S4[(size_t)c * CG + cg] = r;
    }
}

template <int DK, int DV, typename TIn>
cudaError_t launch_typed(const DecodeArgs &a, cudaStream_t stream)
{
    const long long blocks = (long long)a.B * a.H;
    if (blocks == 0) return cudaSuccess;
    if (a.gate == kGateSoftplus)
        decode_step_kernel<DK, DV, TIn, kGateSoftplus><<<(unsigned)blocks, kThreads, 0, stream>>>(
            (const TIn *)a.q, (const TIn *)a.k, (const TIn *)a.v, (const TIn *)a.z, a.A, a.beta,
            a.H, a.state, a.slots, (TIn *)a.o);
    else
        decode_step_kernel<DK, DV, TIn, kGateBounded><<<(unsigned)blocks, kThreads, 0, stream>>>(
            (const TIn *)a.q, (const TIn *)a.k, (const TIn *)a.v, (const TIn *)a.z, a.A, a.beta,
            a.H, a.state, a.slots, (TIn *)a.o);
    return cudaGetLastError();
}

template <int DK, typename TIn>
cudaError_t launch_dv(const DecodeArgs &a, cudaStream_t stream)
{
    switch (a.dv) {
    case 32: return launch_typed<DK, 32, TIn>(a, stream);
    case 64: return launch_typed<DK, 64, TIn>(a, stream);
    case 128: return launch_typed<DK, 128, TIn>(a, stream);
    default: return cudaErrorInvalidValue;
    }
}

template <typename TIn>
cudaError_t launch_dk(const DecodeArgs &a, cudaStream_t stream)
{
    switch (a.dk) {
    case 32: return launch_dv<32, TIn>(a, stream);
    case 64: return launch_dv<64, TIn>(a, stream);
    case 128: return launch_dv<128, TIn>(a, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_decode_step(const DecodeArgs &a, cudaStream_t stream)
{
    return a.bf16 ? launch_dk<__nv_bfloat16>(a, stream) : launch_dk<float>(a, stream);
}

}  // namespace kda
