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
// Persistent CTAs of 2 dv threads walk the (sequence, head) items, as many as
// fit on an SM (two at dk = dv = 128).  While a CTA runs an item's tokens from
// registers, one bulk copy brings the next item's state (dk x dv fp32,
// contiguous in HBM) into shared memory and cp.async brings the rows of its
// first kGroup tokens, so the state stream and the input fetch overlap the token
// arithmetic instead of alternating with it.
// Warp w owns the 16 value columns 16 w .. 16 w + 15 (four float4 column groups)
// for all dk rows: lane (rg, c4) = (lane / 4, lane % 4) holds rows rg, rg + 8,
// ... of column group 4 w + c4 in registers.  Columns of S never mix, so every
// reduction of a token step (vhat and p over the key channels) stays inside a
// warp (three xor shuffles over the row groups), and the token steps need no
// block barrier: each warp runs its own columns' recurrence.  The inputs of
// kGroup tokens at a time, their decays and k.q, are fetched together into
// shared memory (one memory latency and two barriers per group, not per token).
#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_prefill_tc.h"
#include "tc_ptx.cuh"

namespace kda {
namespace {

constexpr int kGroup = 8;   // tokens whose inputs are fetched together
constexpr uint64_t kWaitNs = 2000000000ull;  // limit of the wait for a state copy: 2 s

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) { return __fmul2_rn(a, b); }

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tc::smem_u32(smem_dst)), "l"(gmem_src)
                 : "memory");
}
__device__ __forceinline__ void cp_async4(void *smem_dst, const void *gmem_src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(tc::smem_u32(smem_dst)), "l"(gmem_src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Four consecutive outputs (16-byte aligned for fp32, 8-byte for bf16) in one store.
__device__ __forceinline__ void store4(float *p, float a, float b, float c, float d) {
    *reinterpret_cast<float4 *>(p) = make_float4(a, b, c, d);
}
__device__ __forceinline__ void store4(__nv_bfloat16 *p, float a, float b, float c, float d) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
    uint2 w;
    w.x = *reinterpret_cast<const uint32_t *>(&lo);
    w.y = *reinterpret_cast<const uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(p) = w;
}

template <int DK, int DV, typename TIn>
__global__ void __launch_bounds__(2 * DV, 2)
decode_multi_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k,
                    const TIn *__restrict__ v, const TIn *__restrict__ z,
                    const float *__restrict__ A, const float *__restrict__ beta, int B, int Tq,
                    int H, float *__restrict__ state, const int32_t *__restrict__ slots,
                    const int32_t *__restrict__ num_tokens, int update_state,
                    TIn *__restrict__ o, int32_t *__restrict__ status)
{
    constexpr int CG = DV / 4;        // float4 column groups
    constexpr int NT = 2 * DV;        // 8 row groups x CG column groups
    constexpr int NW = NT / 32;
    constexpr int RPT = DK / 8;       // state rows per thread
    static_assert(CG % 4 == 0 && RPT >= 1, "bad decode tiling");

    __shared__ float sAlphaG[kGroup][DK], sKG[kGroup][DK], sQG[kGroup][DK];
    __shared__ __align__(16) float sVG[kGroup][DV];
    __shared__ float sBetaG[kGroup], sKQG[kGroup];

    extern __shared__ float4 sNext[];   // dk x dv fp32: the state of the CTA's next item
    __shared__ uint64_t full;            // completes when that copy has landed
    // The next item's first kGroup tokens as they are in memory (cp.async during
    // the current item), so that its first group needs no global round trip.
    __shared__ __align__(16) TIn sRawZ[kGroup][DK], sRawK[kGroup][DK], sRawQ[kGroup][DK];
    __shared__ __align__(16) TIn sRawV[kGroup][DV];
    __shared__ float sRawBeta[kGroup];

    const int items = B * H;
    if ((int)blockIdx.x >= items) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rg = lane >> 2, cg = 4 * warp + (lane & 3);
    constexpr uint32_t kStateBytes = DK * DV * 4;
    auto state_of = [&](int w) {
        const int bw = w / H;
        return reinterpret_cast<float4 *>(state + ((size_t)(slots ? slots[bw] : bw) * H + w % H) * DK * DV);
    };
    auto tokens_of = [&](int bw) {
        const int nt = num_tokens ? num_tokens[bw] : Tq;
        return nt < 0 ? 0 : (nt > Tq ? Tq : nt);
    };
    // Every thread copies its share of item w's first group rows (16-byte pieces).
    auto prefetch_inputs = [&](int w) {
        const int bw = w / H, hw = w % H, ng = min(kGroup, tokens_of(bw));
        constexpr int PK = DK * (int)sizeof(TIn) / 16, PV = DV * (int)sizeof(TIn) / 16;
        constexpr int EK = 16 / (int)sizeof(TIn);   // elements per piece
        for (int e = tid; e < ng * PK; e += NT) {
            const int u = e / PK, j = e % PK;
            const size_t row = (((size_t)bw * Tq + u) * H + hw) * DK + (size_t)j * EK;
            cp_async16(&sRawZ[u][j * EK], z + row);
            cp_async16(&sRawK[u][j * EK], k + row);
            cp_async16(&sRawQ[u][j * EK], q + row);
        }
        for (int e = tid; e < ng * PV; e += NT) {
            const int u = e / PV, j = e % PV;
            cp_async16(&sRawV[u][j * EK], v + (((size_t)bw * Tq + u) * H + hw) * DV + (size_t)j * EK);
        }
        if (tid < ng) cp_async4(&sRawBeta[tid], beta + ((size_t)bw * Tq + tid) * H + hw);
        cp_async_commit();
    };
    if (tid == 0) {
        tc::mbar_init(&full, 1);
        tc::fence_mbar_init();
        tc::mbar_arrive_expect_tx(&full, kStateBytes);
        tc::bulk_g2s(sNext, state_of(blockIdx.x), kStateBytes, &full);
    }
    prefetch_inputs(blockIdx.x);
    __syncthreads();
    // The group fetch gives every thread the same key channels in every group
    // (c0 + k NT) and the same value channel (cv), so exp(A) of its channels sits
    // in registers.
    constexpr int TPU = NT >= DK ? NT / DK : 1;   // tokens per pass of the key-channel fetch
    constexpr int CPT = NT >= DK ? 1 : DK / NT;   // key channels per thread
    const int c0 = NT >= DK ? tid % DK : tid, u0 = NT >= DK ? tid / DK : 0;
    const int cv = tid % DV, uv0 = tid / DV;      // NT = 2 DV: two tokens per pass
    int it = 0, issued = 1;                       // items consumed / copies issued (thread 0)
    float eA[CPT];
    // Decays, k, q, v and beta of tokens t .. t + ng - 1 of (b, h) into the group
    // buffers, from the raw rows (first group) or from global memory.
    auto stage_group = [&](int b, int h, int t, int ng, bool raw) {
        for (int u = u0; u < ng; u += TPU) {
            const size_t tu = ((size_t)b * Tq + t + u) * H + h;
#pragma unroll
            for (int k2 = 0; k2 < CPT; ++k2) {
                const int c = c0 + k2 * NT;
                const float zf = to_f32(raw ? sRawZ[u][c] : z[tu * DK + c]);
                sAlphaG[u][c] = expf(gate_log_decay(eA[k2], zf));
                sKG[u][c] = to_f32(raw ? sRawK[u][c] : k[tu * DK + c]);
                sQG[u][c] = to_f32(raw ? sRawQ[u][c] : q[tu * DK + c]);
            }
        }
        for (int u = uv0; u < ng; u += 2)
            sVG[u][cv] = to_f32(raw ? sRawV[u][cv] : v[(((size_t)b * Tq + t + u) * H + h) * DV + cv]);
        if (tid < ng) sBetaG[tid] = raw ? sRawBeta[tid] : beta[((size_t)b * Tq + t + tid) * H + h];
    };
    // k . q of each staged token, one warp each.
    auto kq_group = [&](int ng) {
        for (int u = warp; u < ng; u += NW) {
            float acc = 0.f;
            for (int c = lane; c < DK; c += 32) acc = fmaf(sKG[u][c], sQG[u][c], acc);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (lane == 0) sKQG[u] = acc;
        }
    };

    for (int w = blockIdx.x; w < items; w += gridDim.x, ++it) {
        const int b = w / H, h = w % H;
        const int n_tok = tokens_of(b);
        float4 *S4 = state_of(w);
#pragma unroll
        for (int k2 = 0; k2 < CPT; ++k2) eA[k2] = expf(A[(size_t)h * DK + c0 + k2 * NT]);
        // This item's state, copied into shared memory during the previous item.
        const bool got = tc::mbar_wait(&full, it & 1, tc::globaltimer_ns() + kWaitNs);
        if (!got) atomicCAS(status, 0, (int32_t)KDA_TC_TIMEOUT_CODE);
        cp_async_wait_all();   // this thread's share of the item's first group rows
        if (__syncthreads_or(!got)) break;
        float4 s[RPT];
#pragma unroll
        for (int i = 0; i < RPT; ++i) s[i] = sNext[(rg + 8 * i) * CG + cg];
        if (n_tok > 0) stage_group(b, h, 0, min(kGroup, n_tok), true);
        // Every read of the state buffer and of the raw rows (and of the previous
        // item's group inputs) is done before the next copies land in them.
        tc::fence_proxy_async_smem();
        __syncthreads();
        if (w + (int)gridDim.x < items) {
            if (tid == 0) {
                tc::mbar_arrive_expect_tx(&full, kStateBytes);
                tc::bulk_g2s(sNext, state_of(w + gridDim.x), kStateBytes, &full);
                ++issued;
            }
            prefetch_inputs(w + gridDim.x);
        }
        if (n_tok > 0) {
            kq_group(min(kGroup, n_tok));
            __syncthreads();
        }

        for (int t = 0; t < n_tok; ++t) {
            const int tg = t % kGroup;
            if (tg == 0 && t > 0) {
                // Inputs of tokens t .. t + kGroup - 1 (those that exist), all loads in
                // flight together; the previous group's buffers are no longer read.
                __syncthreads();
                const int ng = min(kGroup, n_tok - t);
                stage_group(b, h, t, ng, false);
                __syncthreads();
                kq_group(ng);
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
                store4(o + vo, fmaf(kq, d.x, p0.x), fmaf(kq, d.y, p0.y), fmaf(kq, d.z, p1.x),
                       fmaf(kq, d.w, p1.y));
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
    // A copy that was issued but not consumed (after a wait gave up) lands before
    // the CTA exits (bounded).
    if (tid == 0)
        for (int d = it; d < issued; ++d) tc::mbar_wait(&full, d & 1, tc::globaltimer_ns() + kWaitNs);
}

template <int DK, int DV, typename TIn>
cudaError_t launch_typed(const DecodeMultiArgs &a, cudaStream_t stream)
{
    const long long items = (long long)a.B * a.H;
    if (items == 0) return cudaSuccess;
    if (items > INT32_MAX) return cudaErrorInvalidValue;
    constexpr int kSmem = DK * DV * 4;
    auto fn = decode_multi_kernel<DK, DV, TIn>;
    // Resident CTAs per SM, once per instantiation (a property of the kernel and the device).
    static int per_sm = 0;
    cudaError_t err;
    if (per_sm == 0) {
        if ((err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem)) != cudaSuccess)
            return err;
        int n = 0;
        if ((err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, 2 * DV, kSmem)) != cudaSuccess)
            return err;
        if (n < 1) return cudaErrorInvalidConfiguration;
        per_sm = n;
    }
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long slots_total = (long long)sms * per_sm;
    const unsigned grid = (unsigned)(items < slots_total ? items : slots_total);
    fn<<<grid, 2 * DV, kSmem, stream>>>(
        (const TIn *)a.q, (const TIn *)a.k, (const TIn *)a.v, (const TIn *)a.z, a.A, a.beta,
        a.B, a.Tq, a.H, a.state, a.slots, a.num_tokens, a.update_state ? 1 : 0, (TIn *)a.o,
        a.status);
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
