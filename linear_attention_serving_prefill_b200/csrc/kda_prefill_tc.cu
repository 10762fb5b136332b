// Chunked KDA prefill on tcgen05 tensor cores (bf16 operands, fp32 accumulate).
//
// Source: "Kimi K3: Architecture, Training, and Million-Token Agentic RL",
// section 3.1 (recurrence), 3.2 (edit order) and 3.3 (chunked prefill: tokens
// of a chunk become matrix products and the state crosses only chunk
// boundaries; the lower-bounded gate keeps a 16-token tile's cumulative
// log-decay in (-80, 0), so the reciprocal factors stay below e^80 and the
// diagonal tiles use the same dense matrix multiply as the off-diagonal ones).
//
// Three launches per call:
//   1. plan:   per-sequence chunk offsets and a longest-first order.
//   2. intra:  one CTA per (64-token chunk, head).  Gate and cumulative
//              log-decay G in fp32, then on the tensor cores
//                A = strictly_lower(Diag(beta) Kt Kh^T), P = lower(Qt Kh^T)
//              (16-token sub-tiles, each with its own reference point), the
//              unit-lower inverse T = (I + A)^-1 on CUDA cores in fp32, and
//                [W | U] = T [Diag(beta) K e^{G} | Diag(beta) V]
//              on the tensor cores.  Writes per (chunk, head) a block of
//              MMA-ready tiles: [W; Q e^{G}], (K e^{G_C - G})^T, P, U, e^{G_C}.
//   3. state:  one persistent CTA per (sequence, head), walking its chunks in
//              order with the fp32 state transposed in tensor memory:
//                D    = S^T [W; Qt]^T              (S^T as a TMEM operand)
//                Dl^T = U^T - D[:, :64]            -> bf16 into TMEM
//                S^T  = S^T Diag(e^{G_C}) + Dl^T Kd   (Kd = K e^{G_C - G})
//                O^T  = D[:, 64:] + Dl^T P^T       -> o
//              Bulk copies stream the per-chunk blocks through a two-stage
//              shared-memory ring.
//
// Within a chunk (tokens r, s; G inclusive from the chunk start):
//   Dl = (I + A)^-1 Diag(beta) (V - Kt S_in) = U - W S_in,
//   O  = Qt S_in + P Dl,   S_out = Diag(e^{G_C}) S_in + Kd^T Dl,
// the recurrence unrolled over the chunk (the derivation is restated in the
// oracle's chunkwise module).
#include <cuda_bf16.h>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_prefill_tc.h"
#include "tc_ptx.cuh"

namespace kda {
namespace {

using namespace tc;

constexpr int kDK = 128, kDV = 128;
constexpr int kChunk = 64;         // state-passing chunk
constexpr int kSub = 16;           // sub-tile with its own decay reference
constexpr uint64_t kWaitNs = 2000000000ull;  // per-wait limit: 2 s

// Per (chunk, head) block written by the intra kernel, read by the state kernel.
constexpr uint32_t kOffWQ = 0;         // [W; Qt] 128 rows x 128 K, swizzled K-major
constexpr uint32_t kOffKd = 32768;     // Kd^T 128 rows (key channel) x 64 K (token)
constexpr uint32_t kOffP = 49152;      // P 64 rows x 64 K
constexpr uint32_t kOffU = 57344;      // U row-major [64][128] bf16
constexpr uint32_t kOffDecay = 73728;  // e^{G_C} [128] fp32
constexpr uint32_t kBlockBytes = 74240;

__device__ __forceinline__ void record_timeout(int32_t *status) {
    atomicCAS(status, 0, (int32_t)KDA_TC_TIMEOUT_CODE);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&p);
}


// ------------------------------------------------------------------- plan --

// chunk_off[n] = sum_{m<n} ceil(L_m / 64); chunk_off[N] = total chunks.
// order[i] = sequence index with the i-th largest length (ties by index)
// when N <= kMaxSorted, else the identity.
constexpr int kPlanThreads = 1024;
constexpr int kMaxSorted = 4096;

__global__ void __launch_bounds__(kPlanThreads)
plan_kernel(const int32_t *__restrict__ cu, int N, int32_t *__restrict__ chunk_off,
            int32_t *__restrict__ order)
{
    __shared__ int32_t part[kPlanThreads];
    const int tid = threadIdx.x;
    const int per = (N + kPlanThreads - 1) / kPlanThreads;
    const int lo = min(N, tid * per), hi = min(N, lo + per);
    int32_t acc = 0;
    for (int n = lo; n < hi; ++n) acc += (cu[n + 1] - cu[n] + kChunk - 1) / kChunk;
    part[tid] = acc;
    __syncthreads();
    for (int off = 1; off < kPlanThreads; off <<= 1) {
        const int32_t v = tid >= off ? part[tid - off] : 0;
        __syncthreads();
        part[tid] += v;
        __syncthreads();
    }
    int32_t run = part[tid] - acc;  // exclusive prefix
    for (int n = lo; n < hi; ++n) {
        chunk_off[n] = run;
        run += (cu[n + 1] - cu[n] + kChunk - 1) / kChunk;
    }
    if (tid == kPlanThreads - 1) chunk_off[N] = part[tid];
    for (int n = tid; n < N; n += kPlanThreads) {
        int rank = n;
        if (N <= kMaxSorted) {
            const int32_t Ln = cu[n + 1] - cu[n];
            rank = 0;
            for (int m = 0; m < N; ++m) {
                const int32_t Lm = cu[m + 1] - cu[m];
                rank += (Lm > Ln) || (Lm == Ln && m < n);
            }
        }
        order[rank] = n;
    }
}

// ------------------------------------------------------------------ intra --

constexpr int kIntraThreads = 128;
// Shared memory of the intra kernel (offsets from a 1024-aligned base).
constexpr uint32_t kIRbig = 0;        // 2 x 160 rows x 128 B: A/P A-operands R^(I)
constexpr uint32_t kIKQ = 40960;      // 2 x 128 rows x 128 B: [Kt_I; Qt_I] per sub-tile
constexpr uint32_t kIBWU = 73728;     // 256 rows x 128 B: [beta K e^G ; beta V]^T
constexpr uint32_t kISmem = 106496;
// Reused after the A/P products are read back:
constexpr uint32_t kIAf = 0;          // fp32 A [64][65]
constexpr uint32_t kITf = 16640;      // fp32 T [64][65]
constexpr uint32_t kIXf = 33280;      // fp32 scratch [32][33]
constexpr uint32_t kITop = kIKQ;      // bf16 T operand 64 rows x 128 B
constexpr int kLd = 65;
// First row of R^(I) in Rbig: 16 * (0 + 1 + ... + I) = 0, 16, 48, 96.
__host__ __device__ constexpr int row_base(int I) { return 8 * I * (I + 1); }

__device__ __forceinline__ int find_seq(const int32_t *chunk_off, int N, int g) {
    int lo = 0, hi = N - 1;  // largest n with chunk_off[n] <= g
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (chunk_off[mid] <= g) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__global__ void __launch_bounds__(kIntraThreads)
intra_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
             const __nv_bfloat16 *__restrict__ v, const __nv_bfloat16 *__restrict__ z,
             const float *__restrict__ A, const float *__restrict__ beta,
             const int32_t *__restrict__ cu, const int32_t *__restrict__ chunk_off, int N, int H,
             uint8_t *__restrict__ blocks, int64_t max_chunks, int32_t *status)
{
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t bar;
    __shared__ uint32_t tbase;
    __shared__ float sBeta[kChunk];
    __shared__ int sAbort;

    const int g = blockIdx.x, h = blockIdx.y, c = threadIdx.x;
    const int total = chunk_off[N];
    if (g >= total) return;
    const int n = find_seq(chunk_off, N, g);
    const int t0 = cu[n] + (g - chunk_off[n]) * kChunk;
    const int len = min(kChunk, cu[n + 1] - t0);
    uint8_t *blk = blocks + ((size_t)h * max_chunks + g) * kBlockBytes;
    const size_t rs = (size_t)H * kDK;                  // token stride (elements)
    const size_t base = (size_t)t0 * rs + (size_t)h * kDK + c;
    const int warp = c >> 5, lane = c & 31;

    if (c == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        sAbort = 0;
    }
    if (c < kChunk) sBeta[c] = c < len ? beta[(size_t)(t0 + c) * H + h] : 0.f;
    if (warp == 0) { tmem_alloc(&tbase, 256); tmem_relinquish(); }

    // Pass 1: gate and cumulative log-decay for key channel c, all 64 rows.
    const float eA = expf(A[(size_t)h * kDK + c]);
    float G[kChunk];
    {
        float acc = 0.f;
#pragma unroll
        for (int r = 0; r < kChunk; ++r) {
            const float zz = r < len ? __bfloat162float(z[base + (size_t)r * rs]) : 0.f;
            acc += r < len ? gate_log_decay(eA, zz) : 0.f;
            G[r] = acc;
        }
    }
    // Sub-tile references m_I = G at the end of sub-tile I-1 (m_0 = 0) and
    // the factors that carry a column operand from its own sub-tile's
    // reference to a later sub-tile's: f[I'][I] = e^{m_I' - m_I} <= 1.
    const float m1 = G[15], m2 = G[31], m3 = G[47], GC = G[63];
    const float mref[4] = {0.f, m1, m2, m3};
    float f[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) f[a][b] = (a > b) ? __expf(mref[a] - mref[b]) : 1.f;
    float emref[4];
#pragma unroll
    for (int I = 0; I < 4; ++I) emref[I] = __expf(mref[I]);
    const float eGC[4] = {__expf(GC - mref[0]), __expf(GC - mref[1]), __expf(GC - mref[2]),
                          __expf(GC - mref[3])};
    __syncthreads();  // sBeta visible

    // Pass 2: scaled operands for channel c.
    uint8_t *sR = sm + kIRbig, *sKQ = sm + kIKQ, *sB = sm + kIBWU;
    uint32_t bufK[4], bufV[4], bufD[4];
#pragma unroll
    for (int r = 0; r < kChunk; ++r) {
        const int I = r / kSub, ri = r % kSub;
        const bool valid = r < len;
        const float kv = valid ? __bfloat162float(k[base + (size_t)r * rs]) : 0.f;
        const float qv = valid ? __bfloat162float(q[base + (size_t)r * rs]) : 0.f;
        const float vv = valid ? __bfloat162float(v[(size_t)(t0 + r) * H * kDV + (size_t)h * kDV + c]) : 0.f;
        const float e1 = __expf(G[r] - mref[I]);   // in [e^-80, 1]
        const float e2 = __expf(mref[I] - G[r]);   // in [1, e^80]
        const float br = sBeta[r];
        // B operand of the A/P products: Kt and Qt scaled to the row sub-tile reference.
        *(__nv_bfloat16 *)(sKQ + sw128_offset(32 * I + ri, c, 128)) = __float2bfloat16_rn(kv * e1);
        *(__nv_bfloat16 *)(sKQ + sw128_offset(32 * I + 16 + ri, c, 128)) = __float2bfloat16_rn(qv * e1);
        // A operands R^(I') for every later sub-tile I' >= I: k e^{m_I' - G_r}.
        const float kb = kv * e2;
#pragma unroll
        for (int Ip = 0; Ip < 4; ++Ip)
            if (Ip >= I)
                *(__nv_bfloat16 *)(sR + sw128_offset(row_base(Ip) + r, c, 160)) =
                    __float2bfloat16_rn(kb * f[Ip][I]);
        // Qt with the chunk-start reference -> rows 64.. of the [W; Qt] tile.
        *(__nv_bfloat16 *)(blk + kOffWQ + sw128_offset(64 + r, c, 128)) =
            __float2bfloat16_rn(qv * e1 * emref[I]);
        // Transposed operands, 8 tokens per 16-byte store.
        const uint32_t hk = __bfloat16_as_ushort(__float2bfloat16_rn(br * kv * e1 * emref[I]));
        const uint32_t hv = __bfloat16_as_ushort(__float2bfloat16_rn(br * vv));
        const uint32_t hd = __bfloat16_as_ushort(__float2bfloat16_rn(kv * e2 * eGC[I]));
        const int slot = (r & 7) >> 1;
        if ((r & 1) == 0) {
            bufK[slot] = hk; bufV[slot] = hv; bufD[slot] = hd;
        } else {
            bufK[slot] |= hk << 16; bufV[slot] |= hv << 16; bufD[slot] |= hd << 16;
        }
        if ((r & 7) == 7) {
            const int r0 = r - 7;
            *(uint4 *)(sB + sw128_offset(c, r0, 256)) = make_uint4(bufK[0], bufK[1], bufK[2], bufK[3]);
            *(uint4 *)(sB + sw128_offset(128 + c, r0, 256)) = make_uint4(bufV[0], bufV[1], bufV[2], bufV[3]);
            *(uint4 *)(blk + kOffKd + sw128_offset(c, r0, 128)) = make_uint4(bufD[0], bufD[1], bufD[2], bufD[3]);
        }
    }
    ((float *)(blk + kOffDecay))[c] = __expf(GC);

    // A/P products on the tensor cores: for sub-tile I, D[s][32I + j] =
    // R^(I)_s . Kt_{16I+j} (j < 16) and R^(I)_s . Qt_{16I+j-16} (j >= 16).
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tb = tbase;
    const uint64_t deadline = globaltimer_ns() + kWaitNs;
    if (c == 0) {
        const uint32_t id = idesc_bf16_f32(64, 32);
#pragma unroll
        for (int I = 0; I < 4; ++I)
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t kb2 = ks >> 2, kin = ks & 3;
                const uint32_t a = smem_u32(sR) + kb2 * 160 * 128 + row_base(I) * 128 + kin * 32;
                const uint32_t b = smem_u32(sKQ) + kb2 * 128 * 128 + 32 * I * 128 + kin * 32;
                mma_ss(tmem_addr(tb, 0, 32 * I), desc_kmajor_sw128(a), desc_kmajor_sw128(b), id, ks > 0);
            }
        mma_commit(&bar);
    }
    if (!mbar_wait(&bar, 0, deadline)) { record_timeout(status); sAbort = 1; }
    tc_fence_after_sync();

    float *Af = (float *)(sm + kIAf), *Tf = (float *)(sm + kITf), *Xf = (float *)(sm + kIXf);
    // Read back (M = 64 layout: row s -> lane 16 * (s / 16) ... warp w lanes 0-15).
    {
        uint32_t rr[32];
        const int s = 16 * warp + lane;
#pragma unroll
        for (int I = 0; I < 4; ++I) {
            tmem_ld32(tmem_addr(tb, 32 * warp, 32 * I), rr);
            tmem_ld_wait();
            if (lane < 16) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int r = 16 * I + j;
                    Af[r * kLd + s] = s < r ? sBeta[r] * __uint_as_float(rr[j]) : 0.f;
                    const float pv = s <= r ? __uint_as_float(rr[16 + j]) : 0.f;
                    *(__nv_bfloat16 *)(blk + kOffP + sw128_offset(r, s, 64)) = __float2bfloat16_rn(pv);
                }
            }
        }
    }
    tc_fence_before_sync();
    __syncthreads();

    // T = (I + A)^-1 by blocks of 16: diagonal blocks by forward substitution,
    // then T_ij = -T_ii A_ij T_jj doubled from 16 to 32 to 64.
    if (c < 64) {
        const int I = c >> 4, j = c & 15, o = 16 * I;
        float col[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float x = (r == j) ? 1.f : 0.f;
#pragma unroll
            for (int s2 = 0; s2 < r; ++s2) x -= Af[(o + r) * kLd + o + s2] * col[s2];
            col[r] = r < j ? 0.f : x;
        }
        for (int r = 0; r < 64; ++r) Tf[r * kLd + o + j] = (r >= o && r < o + 16) ? col[r - o] : 0.f;
    }
    __syncthreads();
    // Level 1: blocks (1,0) and (3,2).  X = A_ij T_jj, then T_ij = -T_ii X.
    for (int e = c; e < 2 * 256; e += kIntraThreads) {
        const int p = e >> 8, r = (e >> 4) & 15, s2 = e & 15;
        const int oi = 32 * p + 16, oj = 32 * p;
        float x = 0.f;
#pragma unroll
        for (int t = 0; t < 16; ++t) x += Af[(oi + r) * kLd + oj + t] * Tf[(oj + t) * kLd + oj + s2];
        Xf[(16 * p + r) * 33 + s2] = x;
    }
    __syncthreads();
    for (int e = c; e < 2 * 256; e += kIntraThreads) {
        const int p = e >> 8, r = (e >> 4) & 15, s2 = e & 15;
        const int oi = 32 * p + 16, oj = 32 * p;
        float x = 0.f;
#pragma unroll
        for (int t = 0; t < 16; ++t) x += Tf[(oi + r) * kLd + oi + t] * Xf[(16 * p + t) * 33 + s2];
        Tf[(oi + r) * kLd + oj + s2] = -x;
    }
    __syncthreads();
    // Level 2: block rows 32..63, columns 0..31.
    for (int e = c; e < 1024; e += kIntraThreads) {
        const int r = e >> 5, s2 = e & 31;
        float x = 0.f;
#pragma unroll 8
        for (int t = 0; t < 32; ++t) x += Af[(32 + r) * kLd + t] * Tf[t * kLd + s2];
        Xf[r * 33 + s2] = x;
    }
    __syncthreads();
    for (int e = c; e < 1024; e += kIntraThreads) {
        const int r = e >> 5, s2 = e & 31;
        float x = 0.f;
#pragma unroll 8
        for (int t = 0; t < 32; ++t) x += Tf[(32 + r) * kLd + 32 + t] * Xf[t * 33 + s2];
        Tf[(32 + r) * kLd + s2] = -x;
    }
    __syncthreads();
    // T as the bf16 A operand of the W/U product (64 rows x 64 K).
    uint8_t *sT = sm + kITop;
    for (int e = c; e < 64 * 64; e += kIntraThreads) {
        const int r = e >> 6, s2 = e & 63;
        *(__nv_bfloat16 *)(sT + sw128_offset(r, s2, 64)) = __float2bfloat16_rn(Tf[r * kLd + s2]);
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (c == 0 && !sAbort) {
        const uint32_t id = idesc_bf16_f32(64, 256);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_ss(tmem_addr(tb, 0, 0), desc_kmajor_sw128(smem_u32(sT) + ks * 32),
                   desc_kmajor_sw128(smem_u32(sB) + ks * 32), id, ks > 0);
        mma_commit(&bar);
    }
    bool ok = !sAbort && mbar_wait(&bar, 1, deadline + kWaitNs);
    if (!ok && !sAbort) record_timeout(status);
    tc_fence_after_sync();
    if (ok) {
        // W -> rows 0..63 of the [W; Qt] tile, U -> row-major U.
        uint32_t rr[32];
        const int r = 16 * warp + lane;
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
            tmem_ld32(tmem_addr(tb, 32 * warp, 32 * q4), rr);
            tmem_ld_wait();
            if (lane < 16) {
#pragma unroll
                for (int cc = 0; cc < 32; cc += 8) {
                    const uint4 w4 = make_uint4(pack_bf16(__uint_as_float(rr[cc]), __uint_as_float(rr[cc + 1])),
                                                pack_bf16(__uint_as_float(rr[cc + 2]), __uint_as_float(rr[cc + 3])),
                                                pack_bf16(__uint_as_float(rr[cc + 4]), __uint_as_float(rr[cc + 5])),
                                                pack_bf16(__uint_as_float(rr[cc + 6]), __uint_as_float(rr[cc + 7])));
                    const int col = 32 * q4 + cc;
                    if (col < 128)
                        *(uint4 *)(blk + kOffWQ + sw128_offset(r, col, 128)) = w4;
                    else
                        *(uint4 *)(blk + kOffU + (size_t)(r * 128 + col - 128) * 2) = w4;
                }
            }
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, 256);
}

// ------------------------------------------------------------------ state --

constexpr int kStateThreads = 320;       // WG0: warps 0-3, WG1: warps 4-7, load: 8, mma: 9
constexpr uint32_t kStageBytes = 75776;  // block rounded up to 1 KiB
constexpr int kStages = 2;
constexpr uint32_t kStateSmem = kStages * kStageBytes + 1024;
// TMEM columns
constexpr uint32_t kTS = 0, kTSbf = 128, kTDl = 192, kTD1 = 256;  // D1 double buffer: 256, 384

struct StateBars {
    uint64_t full[kStages], empty[kStages];
    uint64_t mma1, dl_ready, sbf_ready;
    uint64_t mma2[2], d1_free[2];
};

__global__ void __launch_bounds__(kStateThreads, 1)
state_kernel(const int32_t *__restrict__ cu, const int32_t *__restrict__ chunk_off,
             const int32_t *__restrict__ order, int N, int H,
             const uint8_t *__restrict__ blocks, int64_t max_chunks,
             const float *S0, float *Sf, __nv_bfloat16 *__restrict__ o, int32_t *status)
{
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
    __shared__ StateBars bars;
    __shared__ uint32_t tbase;
    __shared__ volatile int sAbort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = order[blockIdx.x / H], h = blockIdx.x % H;
    const int tbeg = cu[n], tend = cu[n + 1];
    const int nch = chunk_off[n + 1] - chunk_off[n];
    const size_t sbase = ((size_t)n * H + h) * kDK * kDV;

    if (nch == 0) {  // empty sequence: the state passes through
        if (Sf)
            for (int e = tid; e < kDK * kDV; e += kStateThreads) Sf[sbase + e] = S0 ? S0[sbase + e] : 0.f;
        return;
    }
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) { mbar_init(&bars.full[s], 1); mbar_init(&bars.empty[s], 129); }
        mbar_init(&bars.mma1, 1);
        mbar_init(&bars.dl_ready, 128);
        mbar_init(&bars.sbf_ready, 128);
        for (int b = 0; b < 2; ++b) { mbar_init(&bars.mma2[b], 1); mbar_init(&bars.d1_free[b], 128); }
        fence_mbar_init();
        sAbort = 0;
    }
    if (warp == 0) { tmem_alloc(&tbase, 512); tmem_relinquish(); }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tb = tbase;
    const uint8_t *blk0 = blocks + ((size_t)h * max_chunks + chunk_off[n]) * kBlockBytes;

    if (warp == 8) {
        // ---- loader: one bulk copy per chunk block into the stage ring ----
        if (lane == 0) {
            int issued = 0;
            for (int c = 0; c < nch && !sAbort; ++c) {
                const int s = c % kStages;
                if (c >= kStages &&
                    !mbar_wait(&bars.empty[s], ((c / kStages) - 1) & 1, globaltimer_ns() + kWaitNs)) {
                    record_timeout(status); sAbort = 1; break;
                }
                mbar_arrive_expect_tx(&bars.full[s], kBlockBytes);
                bulk_g2s(sm + s * kStageBytes, blk0 + (size_t)c * kBlockBytes, kBlockBytes, &bars.full[s]);
                ++issued;
            }
            // Drain: every issued copy has landed before the CTA may exit.
            for (int c = max(0, issued - kStages); c < issued; ++c)
                mbar_wait(&bars.full[c % kStages], (c / kStages) & 1, globaltimer_ns() + kWaitNs);
        }
    } else if (warp == 9) {
        // ---- MMA issuer ----
        if (lane == 0) {
            const uint32_t id128 = idesc_bf16_f32(128, 128), id64 = idesc_bf16_f32(128, 64);
            int c = 0;
            for (; c < nch && !sAbort; ++c) {
                const int s = c % kStages, b = c & 1;
                const uint32_t st = smem_u32(sm + s * kStageBytes);
                const uint32_t d1 = tmem_addr(tb, 0, kTD1 + 128 * b);
                bool ok = mbar_wait(&bars.full[s], (c / kStages) & 1, globaltimer_ns() + kWaitNs) &&
                          mbar_wait(&bars.sbf_ready, c & 1, globaltimer_ns() + kWaitNs) &&
                          (c < 2 || mbar_wait(&bars.d1_free[b], ((c >> 1) - 1) & 1, globaltimer_ns() + kWaitNs));
                if (!ok) { record_timeout(status); sAbort = 1; break; }
                tc_fence_after_sync();
                // D1 = S^T [W; Qt]^T  (M = dv, N = 128 tokens-by-two, K = dk)
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_ts(d1, tmem_addr(tb, 0, kTSbf + 8 * ks),
                           desc_kmajor_sw128(st + kOffWQ + (ks >> 2) * 128 * 128 + (ks & 3) * 32),
                           id128, ks > 0);
                mma_commit(&bars.mma1);
                if (!mbar_wait(&bars.dl_ready, c & 1, globaltimer_ns() + kWaitNs)) {
                    record_timeout(status); sAbort = 1; break;
                }
                tc_fence_after_sync();
                // S^T += Dl^T Kd (N = dk, K = 64 tokens); O^T += Dl^T P^T (N = 64, K = 64)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_ts(tmem_addr(tb, 0, kTS), tmem_addr(tb, 0, kTDl + 8 * ks),
                           desc_kmajor_sw128(st + kOffKd + ks * 32), id128, true);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_ts(d1 + 64, tmem_addr(tb, 0, kTDl + 8 * ks),
                           desc_kmajor_sw128(st + kOffP + ks * 32), id64, true);
                mma_commit(&bars.mma2[b]);
                mma_commit(&bars.empty[s]);
            }
            // Drain: wait for the last committed MMAs before exit.
            if (c > 0) mbar_wait(&bars.mma2[(c - 1) & 1], ((c - 1) >> 1) & 1, globaltimer_ns() + kWaitNs);
        }
    } else if (warp < 4) {
        // ---- WG0: the delta and the state passes; thread j = value channel j ----
        const int j = tid;
        const uint32_t lq = 32 * warp;
        uint32_t r32[32];
        // Initial state: S^T row j = column j of S0; bf16 copy and pre-decay.
        bool ok = true;
        const float *dec0 = nullptr;
        if (S0) {
            ok = mbar_wait(&bars.full[0], 0, globaltimer_ns() + kWaitNs);
            if (!ok) { record_timeout(status); sAbort = 1; }
            dec0 = (const float *)(sm + kOffDecay);
        }
        for (int q4 = 0; q4 < 4 && ok; ++q4) {
            float sv[32];
#pragma unroll
            for (int i = 0; i < 32; ++i)
                sv[i] = S0 ? S0[sbase + (size_t)(32 * q4 + i) * kDV + j] : 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) r32[i] = __float_as_uint(S0 ? sv[i] * dec0[32 * q4 + i] : 0.f);
            tmem_st32(tmem_addr(tb, lq, kTS + 32 * q4), r32);
            uint32_t sb[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) sb[i] = pack_bf16(sv[2 * i], sv[2 * i + 1]);
            tmem_st16(tmem_addr(tb, lq, kTSbf + 16 * q4), sb);
        }
        tmem_st_wait();
        tc_fence_before_sync();
        mbar_arrive(&bars.sbf_ready);

        for (int c = 0; c < nch && !sAbort; ++c) {
            const int s = c % kStages, b = c & 1;
            const uint8_t *st = sm + s * kStageBytes;
            if (!mbar_wait(&bars.full[s], (c / kStages) & 1, globaltimer_ns() + kWaitNs) ||
                !mbar_wait(&bars.mma1, c & 1, globaltimer_ns() + kWaitNs)) {
                record_timeout(status); sAbort = 1; break;
            }
            tc_fence_after_sync();
            // Dl^T[j][r] = U[r][j] - D1[j][r], r < 64 -> bf16 pairs into TMEM.
            const __nv_bfloat16 *U = (const __nv_bfloat16 *)(st + kOffU);
            uint32_t dl[32];
#pragma unroll
            for (int hlf = 0; hlf < 2; ++hlf) {
                tmem_ld32(tmem_addr(tb, lq, kTD1 + 128 * b + 32 * hlf), r32);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const int r = 32 * hlf + i;
                    const float d0 = __bfloat162float(U[r * kDV + j]) - __uint_as_float(r32[i]);
                    const float d1v = __bfloat162float(U[(r + 1) * kDV + j]) - __uint_as_float(r32[i + 1]);
                    dl[16 * hlf + (i >> 1)] = pack_bf16(d0, d1v);
                }
            }
            tmem_st32(tmem_addr(tb, lq, kTDl), dl);
            tmem_st_wait();
            tc_fence_before_sync();
            mbar_arrive(&bars.dl_ready);
            mbar_arrive(&bars.empty[s]);  // done with U of this stage

            if (!mbar_wait(&bars.mma2[b], (c >> 1) & 1, globaltimer_ns() + kWaitNs)) {
                record_timeout(status); sAbort = 1; break;
            }
            tc_fence_after_sync();
            const bool last = (c + 1 == nch);
            const float *dec = nullptr;
            if (!last) {
                const int s1 = (c + 1) % kStages;
                if (!mbar_wait(&bars.full[s1], ((c + 1) / kStages) & 1, globaltimer_ns() + kWaitNs)) {
                    record_timeout(status); sAbort = 1; break;
                }
                dec = (const float *)(sm + s1 * kStageBytes + kOffDecay);
            }
            // S_out -> bf16 copy for the next chunk, and pre-decayed fp32 state.
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                tmem_ld32(tmem_addr(tb, lq, kTS + 32 * q4), r32);
                tmem_ld_wait();
                if (last) {
                    if (Sf) {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            Sf[sbase + (size_t)(32 * q4 + i) * kDV + j] = __uint_as_float(r32[i]);
                    }
                    continue;
                }
                uint32_t sb[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    sb[i] = pack_bf16(__uint_as_float(r32[2 * i]), __uint_as_float(r32[2 * i + 1]));
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    r32[i] = __float_as_uint(__uint_as_float(r32[i]) * dec[32 * q4 + i]);
                tmem_st32(tmem_addr(tb, lq, kTS + 32 * q4), r32);
                tmem_st16(tmem_addr(tb, lq, kTSbf + 16 * q4), sb);
            }
            if (!last) {
                tmem_st_wait();
                tc_fence_before_sync();
                mbar_arrive(&bars.sbf_ready);
            }
        }
    } else {
        // ---- WG1: outputs; thread j = value channel j ----
        const int j = tid - 128;
        const uint32_t lq = 32 * (warp - 4);
        uint32_t r32[32];
        for (int c = 0; c < nch && !sAbort; ++c) {
            const int b = c & 1;
            if (!mbar_wait(&bars.mma2[b], (c >> 1) & 1, globaltimer_ns() + kWaitNs)) {
                record_timeout(status); sAbort = 1; break;
            }
            tc_fence_after_sync();
            const int t0 = tbeg + c * kChunk;
            const int len = min(kChunk, tend - t0);
#pragma unroll
            for (int hlf = 0; hlf < 2; ++hlf) {
                tmem_ld32(tmem_addr(tb, lq, kTD1 + 128 * b + 64 + 32 * hlf), r32);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int r = 32 * hlf + i;
                    if (r < len)
                        o[((size_t)(t0 + r) * H + h) * kDV + j] = __float2bfloat16_rn(__uint_as_float(r32[i]));
                }
            }
            tc_fence_before_sync();
            mbar_arrive(&bars.d1_free[b]);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, 512);
}

}  // namespace

size_t tc_workspace_bytes(int32_t total_tokens, int32_t num_seqs, int32_t H)
{
    if (num_seqs <= 0) return 0;
    const int64_t max_chunks = ((int64_t)total_tokens + 63LL * num_seqs) / kChunk;
    const size_t plan = (((size_t)(2 * num_seqs + 2) * sizeof(int32_t)) + 1023) & ~(size_t)1023;
    return plan + (size_t)H * max_chunks * kBlockBytes;
}

cudaError_t launch_prefill_tensor_core(const PrefillArgs &a, cudaStream_t stream)
{
    if (a.dk != kDK || a.dv != kDV || !a.bf16) return cudaErrorInvalidValue;
    const int64_t max_chunks = ((int64_t)a.total_tokens + 63LL * a.num_seqs) / kChunk;
    int32_t *chunk_off = (int32_t *)a.workspace;
    int32_t *order = chunk_off + a.num_seqs + 1;
    const size_t plan = (((size_t)(2 * a.num_seqs + 2) * sizeof(int32_t)) + 1023) & ~(size_t)1023;
    uint8_t *blocks = (uint8_t *)a.workspace + plan;
    cudaError_t err;

    err = cudaFuncSetAttribute(intra_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)(kISmem + 1024));
    if (err != cudaSuccess) return err;
    err = cudaFuncSetAttribute(state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kStateSmem);
    if (err != cudaSuccess) return err;

    a.mark(0, stream);
    plan_kernel<<<1, kPlanThreads, 0, stream>>>(a.cu_seqlens, a.num_seqs, chunk_off, order);
    a.mark(1, stream);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;

    const int ismem = kISmem + 1024;
    if (max_chunks > 0) {
        dim3 grid((unsigned)max_chunks, (unsigned)a.H);
        intra_kernel<<<grid, kIntraThreads, ismem, stream>>>(
            (const __nv_bfloat16 *)a.q, (const __nv_bfloat16 *)a.k, (const __nv_bfloat16 *)a.v,
            (const __nv_bfloat16 *)a.z, a.A, a.beta, a.cu_seqlens, chunk_off, a.num_seqs, a.H,
            blocks, max_chunks, a.status);
        err = cudaGetLastError();
        if (err != cudaSuccess) return err;
    }
    a.mark(2, stream);
    state_kernel<<<(unsigned)(a.num_seqs * a.H), kStateThreads, kStateSmem, stream>>>(
        a.cu_seqlens, chunk_off, order, a.num_seqs, a.H, blocks, max_chunks, a.initial_state,
        a.final_state, (__nv_bfloat16 *)a.o, a.status);
    a.mark(3, stream);
    return cudaGetLastError();
}

}  // namespace kda
