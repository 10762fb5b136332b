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
//   2. intra:  persistent, one CTA per SM over the (64-token chunk, head) items.  Gate and cumulative
//              log-decay G in fp32, then on the tensor cores
//                A = strictly_lower(Diag(beta) Kt Kh^T), P = lower(Qt Kh^T)
//              (16-token sub-tiles, each with its own reference point), the
//              unit-lower inverse T = (I + A)^-1 on CUDA cores in fp32, and
//                [W | U] = T [Diag(beta) K e^{G} | Diag(beta) V]
//              on the tensor cores.  Writes per (chunk, head) a block of
//              MMA-ready tiles: [W; Q e^{G}], (K e^{G_C - G})^T, P, U, e^{G_C}.
//   3. state:  one persistent CTA per (sequence, head), walking its chunks in
//              order with the fp32 state transposed in tensor memory (two
//              epilogue warpgroups split every pass by rows / key channels):
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
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <mutex>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_prefill_tc.h"
#include "tc_ptx.cuh"

namespace kda {
namespace {

using namespace tc;

constexpr int kDK = 128, kDV = 128;
constexpr int kChunk = 64;         // state-passing chunk
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
// ckpt_off[n] = sum_{m<n} L_m / every (checkpoint rows), when every > 0.
// order[i] = sequence index with the i-th largest length (ties by index)
// when N <= kMaxSorted, else the identity.
constexpr int kPlanThreads = 1024;
constexpr int kMaxSorted = 4096;

__global__ void __launch_bounds__(kPlanThreads)
plan_kernel(const int32_t *__restrict__ cu, int N, int every, int32_t *__restrict__ chunk_off,
            int32_t *__restrict__ ckpt_off, int32_t *__restrict__ order)
{
    __shared__ int32_t part[2][kPlanThreads];
    const int tid = threadIdx.x;
    const int per = (N + kPlanThreads - 1) / kPlanThreads;
    const int lo = min(N, tid * per), hi = min(N, lo + per);
    int32_t acc = 0, acck = 0;
    for (int n = lo; n < hi; ++n) {
        const int32_t L = cu[n + 1] - cu[n];
        acc += (L + kChunk - 1) / kChunk;
        acck += every > 0 ? L / every : 0;
    }
    part[0][tid] = acc;
    part[1][tid] = acck;
    __syncthreads();
    for (int off = 1; off < kPlanThreads; off <<= 1) {
        const int32_t v0 = tid >= off ? part[0][tid - off] : 0;
        const int32_t v1 = tid >= off ? part[1][tid - off] : 0;
        __syncthreads();
        part[0][tid] += v0;
        part[1][tid] += v1;
        __syncthreads();
    }
    int32_t run = part[0][tid] - acc, runk = part[1][tid] - acck;  // exclusive prefixes
    for (int n = lo; n < hi; ++n) {
        const int32_t L = cu[n + 1] - cu[n];
        chunk_off[n] = run;
        ckpt_off[n] = runk;
        run += (L + kChunk - 1) / kChunk;
        runk += every > 0 ? L / every : 0;
    }
    if (tid == kPlanThreads - 1) {
        chunk_off[N] = part[0][tid];
        ckpt_off[N] = part[1][tid];
    }
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

// Persistent: one CTA per SM walks (chunk, head) items b, b + gridDim.x, ...;
// item w is chunk w / H of head w % H.  While an item is computed, warp 0
// prefetches the next item's raw k, q, v, z rows (256 B each) into the other
// stage of a two-stage ring with bulk copies, and its beta values with
// cp.async.  Thread (cp, q8) owns channels 2 cp, 2 cp + 1 of the eight rows
// 8 q8 .. 8 q8 + 7 (q8 = warp / 2), inside sub-tile I = q8 / 2, so the
// sub-tile index is uniform across a warp.
constexpr int kIntraCompute = 512;
constexpr int kIntraThreads = kIntraCompute;
constexpr uint32_t kRawTile = kChunk * kDK * 2;    // one [64][128] bf16 tile, 16 KiB
constexpr uint32_t kRawStage = 4 * kRawTile;       // k, q, v, z
constexpr uint32_t kRawK = 0, kRawQ = kRawTile, kRawV = 2 * kRawTile, kRawZ = 3 * kRawTile;
// Shared memory (offsets from a 1024-aligned base).
constexpr uint32_t kIRaw = 0;                      // 2 raw stages
// A operands of the A/P products, R^(I) = k e^{m_I - G} scaled to sub-tile I's
// reference, stacked in pairs for M = 128 products: pair p holds R^(2p+1) in rows
// 0..63 and R^(2p) in rows 64..127, one 128-row x 128-byte sub-block per 64-wide
// K half.  Rows that are never valid (R^(I) beyond row 16 I + 15) sit at the ends
// of some sub-blocks, so the next buffer starts inside that tail: the product
// reads whatever is there into rows it discards, and nobody writes them.
constexpr uint32_t kIRbig = 2 * kRawStage;
__host__ __device__ constexpr uint32_t r_sub(int p, int kb) {
    return p == 0 ? (kb == 0 ? 0u : 10240u) : (kb == 0 ? 20480u : 34816u);
}
constexpr uint32_t kIKQ = kIRbig + 49152;          // [Kt_I; Qt_I] per sub-tile, then [bK e^G; bV]^T
constexpr uint32_t kISmem = kIKQ + 32768;
// Reused inside Rbig once the A/P products are read back:
constexpr uint32_t kIAf = kIRbig;                  // fp32 A [64][65]
constexpr uint32_t kITf = kIRbig + 16640;          // fp32 T [64][65]
constexpr uint32_t kIXf = kIRbig + 33280;          // fp32 scratch [32][33]
constexpr int kLd = 65;
// Row block of sub-tile I inside its pair: 0 for the odd tile, 64 for the even one.
__host__ __device__ constexpr int pair_slot_row(int I) { return (I & 1) ? 0 : 64; }

struct IntraItem { int t0, len, g, h; };

// One 3-D tile load: the box {128 channels, 1 head, 64 tokens} at (0, h, t0)
// of a [T][H][128] bf16 tensor; rows past T arrive as zeros.
__device__ __forceinline__ void tma_rows(void *smem_dst, const CUtensorMap *map, int h, int t0,
                                         uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];"
        ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(h), "r"(t0),
          "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void compute_sync() { __syncthreads(); }

__device__ __forceinline__ void cp_async_4(void *smem_dst, const void *gmem_src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ int find_seq(const int32_t *chunk_off, int N, int g) {
    int lo = 0, hi = N - 1;  // largest n with chunk_off[n] <= g
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (chunk_off[mid] <= g) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ float2 ld_bf16x2_smem(const uint8_t *base, uint32_t off) {
    return __bfloat1622float2(*(const __nv_bfloat162 *)(base + off));
}

__device__ __forceinline__ uint32_t bf16_bits(float x) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// The gate with the fast exponential and division (a few ulp; the bf16 path's
// tolerance is far looser).  Limits as in gate_log_decay: exp(A) z -> +inf gives
// g_min, -> -inf gives 0 (1 / +inf through the fast division is 0).
__device__ __forceinline__ float gate_log_decay_fast(float expA, float z) {
    return __fdividef(kGMin, 1.0f + __expf(-expA * z));
}

__global__ void __launch_bounds__(kIntraThreads, 1)
intra_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_z,
             const float *__restrict__ A, const float *__restrict__ beta,
             const int32_t *__restrict__ cu, const int32_t *__restrict__ chunk_off, int N, int H,
             uint8_t *__restrict__ blocks, int64_t max_chunks, int32_t *status)
{
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t full[2], mma_bar;
    __shared__ uint32_t tbase;
    __shared__ IntraItem info[2];
    __shared__ float sBeta[2][kChunk];
    __shared__ float sTot[8][kDK];
    __shared__ volatile int sAbort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int total_items = chunk_off[N] * H;
    if ((int)blockIdx.x >= total_items) return;
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) mbar_init(&full[s], 1);
        mbar_init(&mma_bar, 1);
        fence_mbar_init();
        sAbort = 0;
    }
    if (warp == 0) { tmem_alloc(&tbase, 256); tmem_relinquish(); }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tb = tbase;

    // Warp 0: request item wn into stage sn (raw rows by bulk copy, beta by cp.async).
    auto issue = [&](int wn, int sn) {
        const int g = wn / H, h = wn % H;
        const int n = find_seq(chunk_off, N, g);
        const int t0 = cu[n] + (g - chunk_off[n]) * kChunk;
        const int len = min(kChunk, cu[n + 1] - t0);
        for (int r = lane; r < kChunk; r += 32) {
            if (r < len) cp_async_4(&sBeta[sn][r], beta + (size_t)(t0 + r) * H + h);
            else sBeta[sn][r] = 0.f;
        }
        cp_async_commit();
        if (lane == 0) {
            // The stage's previous item staged W, U and Kd^T in it for bulk stores:
            // all but the newest bulk group (this item's Kd^T) have finished reading.
            bulk_wait_read<1>();
            info[sn] = IntraItem{t0, len, g, h};
            mbar_arrive_expect_tx(&full[sn], kRawStage);
            uint8_t *stn = sm + kIRaw + sn * kRawStage;
            tma_rows(stn + kRawK, &tm_k, h, t0, &full[sn]);
            tma_rows(stn + kRawQ, &tm_q, h, t0, &full[sn]);
            tma_rows(stn + kRawV, &tm_v, h, t0, &full[sn]);
            tma_rows(stn + kRawZ, &tm_z, h, t0, &full[sn]);
        }
        __syncwarp();
    };
    if (warp == 0) issue(blockIdx.x, 0);
    int issued = 1;  // items requested so far (meaningful in warp 0)

    {
        // Thread (cp, q8): channels c0 = 2 cp and c0 + 1, rows 8 q8 .. 8 q8 + 7, sub-tile I.
        const int cp = ((warp & 1) << 5) | lane, c0 = 2 * cp, q8 = warp >> 1, I = q8 >> 1;
        uint32_t mma_count = 0;
        int it = 0;
        for (int w = blockIdx.x; w < total_items && !sAbort; w += gridDim.x, ++it) {
            const int s = it & 1;
            if (warp == 0) cp_async_wait_all();  // this item's beta values (issued one item ago)
            if (!mbar_wait(&full[s], (it >> 1) & 1, globaltimer_ns() + kWaitNs)) {
                if (tid == 0) record_timeout(status);
                sAbort = 1;
                break;
            }
            const IntraItem inf = info[s];
            const int len = inf.len, h = inf.h;
            const uint8_t *st = sm + kIRaw + s * kRawStage;
            uint8_t *blk = blocks + ((size_t)h * max_chunks + inf.g) * kBlockBytes;
            const float2 eA = make_float2(__expf(A[(size_t)h * kDK + c0]), __expf(A[(size_t)h * kDK + c0 + 1]));

            // Pass 1: gate and cumulative log-decay of channels c0, c0 + 1 over the
            // eight rows, then relative to the sub-tile start: L_r = G_r - m_I.
            float2 L[8];
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = 8 * q8 + i;
                if (r < len) {
                    const float2 zz = ld_bf16x2_smem(st, kRawZ + r * 256 + 4 * cp);
                    acc.x += gate_log_decay_fast(eA.x, zz.x);
                    acc.y += gate_log_decay_fast(eA.y, zz.y);
                }
                L[i] = acc;
            }
            sTot[q8][c0] = acc.x;
            sTot[q8][c0 + 1] = acc.y;
            compute_sync();
            if (q8 & 1) {
                const float ox = sTot[q8 - 1][c0], oy = sTot[q8 - 1][c0 + 1];
#pragma unroll
                for (int i = 0; i < 8; ++i) { L[i].x += ox; L[i].y += oy; }
            }
            // Sub-tile references m_J = G at the end of sub-tile J - 1 (m_0 = 0), G_C.
            float2 mref[5];
            mref[0] = make_float2(0.f, 0.f);
#pragma unroll
            for (int J = 0; J < 4; ++J)
                mref[J + 1] = make_float2(mref[J].x + sTot[2 * J][c0] + sTot[2 * J + 1][c0],
                                          mref[J].y + sTot[2 * J][c0 + 1] + sTot[2 * J + 1][c0 + 1]);
            const float2 mI = I == 0 ? mref[0] : I == 1 ? mref[1] : I == 2 ? mref[2] : mref[3];
            const float2 GC = mref[4];
            const float2 emI = make_float2(__expf(mI.x), __expf(mI.y));
            const float2 egc = make_float2(__expf(GC.x - mI.x), __expf(GC.y - mI.y));
            // fac[Ip] = e^{m_Ip - m_I} carries a column operand from sub-tile I's
            // reference to a later sub-tile's (1 for Ip = I).
            float2 fac[4];
#pragma unroll
            for (int Ip = 0; Ip < 4; ++Ip)
                fac[Ip] = Ip > I ? make_float2(__expf(mref[Ip].x - mI.x), __expf(mref[Ip].y - mI.y))
                                 : make_float2(1.f, 1.f);

            // Pass 2: scaled operands of channels c0, c0 + 1 for the eight rows.
            uint8_t *sR = sm + kIRbig, *sKQ = sm + kIKQ;
            uint32_t pk0[4], pk1[4], pv0[4], pv1[4], kd0[4], kd1[4];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = 8 * q8 + i, ri = r & 15;
                const bool valid = r < len;
                const float2 kv = valid ? ld_bf16x2_smem(st, kRawK + r * 256 + 4 * cp) : make_float2(0.f, 0.f);
                const float2 qv = valid ? ld_bf16x2_smem(st, kRawQ + r * 256 + 4 * cp) : make_float2(0.f, 0.f);
                const float2 vv = valid ? ld_bf16x2_smem(st, kRawV + r * 256 + 4 * cp) : make_float2(0.f, 0.f);
                const float2 e1 = make_float2(__expf(L[i].x), __expf(L[i].y));    // in [e^-80, 1]
                const float2 e2 = make_float2(__expf(-L[i].x), __expf(-L[i].y));  // in [1, e^80]
                const float br = sBeta[s][r];
                // B rows of pair I / 2: [Kt_odd; Qt_odd; Kt_even; Qt_even], 16 rows each.
                const int brow = 64 * (I >> 1) + ((I & 1) ? 0 : 32) + ri;
                *(uint32_t *)(sKQ + sw128_offset(brow, c0, 128)) = pack_bf16(kv.x * e1.x, kv.y * e1.y);
                *(uint32_t *)(sKQ + sw128_offset(brow + 16, c0, 128)) = pack_bf16(qv.x * e1.x, qv.y * e1.y);
                const float2 kb = make_float2(kv.x * e2.x, kv.y * e2.y);
#pragma unroll
                for (int Ip = 0; Ip < 4; ++Ip)
                    if (Ip >= I)
                        *(uint32_t *)(sR + r_sub(Ip >> 1, c0 >> 6) +
                                      sw128_offset(pair_slot_row(Ip) + r, c0 & 63, 128)) =
                            pack_bf16(kb.x * fac[Ip].x, kb.y * fac[Ip].y);
                *(uint32_t *)(blk + kOffWQ + sw128_offset(64 + r, c0, 128)) =
                    pack_bf16(qv.x * e1.x * emI.x, qv.y * e1.y * emI.y);
                const uint32_t hk0 = bf16_bits(br * kv.x * e1.x * emI.x), hk1 = bf16_bits(br * kv.y * e1.y * emI.y);
                const uint32_t hv0 = bf16_bits(br * vv.x), hv1 = bf16_bits(br * vv.y);
                const uint32_t hd0 = bf16_bits(kb.x * egc.x), hd1 = bf16_bits(kb.y * egc.y);
                if ((i & 1) == 0) {
                    pk0[i >> 1] = hk0; pk1[i >> 1] = hk1; pv0[i >> 1] = hv0; pv1[i >> 1] = hv1;
                    kd0[i >> 1] = hd0; kd1[i >> 1] = hd1;
                } else {
                    pk0[i >> 1] |= hk0 << 16; pk1[i >> 1] |= hk1 << 16;
                    pv0[i >> 1] |= hv0 << 16; pv1[i >> 1] |= hv1 << 16;
                    kd0[i >> 1] |= hd0 << 16; kd1[i >> 1] |= hd1 << 16;
                }
            }
            // (K e^{G_C - G})^T is staged in the item's raw z tile (dead after pass 1)
            // as the exact image of its block region, then bulk-stored.
            uint8_t *stw = sm + kIRaw + s * kRawStage;
            *(uint4 *)(stw + kRawZ + sw128_offset(c0, 8 * q8, 128)) = make_uint4(kd0[0], kd0[1], kd0[2], kd0[3]);
            *(uint4 *)(stw + kRawZ + sw128_offset(c0 + 1, 8 * q8, 128)) = make_uint4(kd1[0], kd1[1], kd1[2], kd1[3]);
            if (q8 == 0) {
                ((float *)(blk + kOffDecay))[c0] = __expf(GC.x);
                ((float *)(blk + kOffDecay))[c0 + 1] = __expf(GC.y);
            }

            // A/P products: D[s][32 I + j] = R^(I)_s . Kt_{16I+j} (j < 16) and . Qt (j >= 16).
            fence_proxy_async_smem();
            tc_fence_before_sync();
            compute_sync();
            tc_fence_after_sync();
            if (tid == 0) {
                bulk_s2g(blk + kOffKd, stw + kRawZ, 16384);
                bulk_commit();
                // Pair p: D[:, 64p .. 64p+63] = [R^(2p+1); R^(2p)] [B_(2p+1); B_(2p)]^T
                // (M = 128, N = 64); the wanted blocks are rows 0..63 x columns 0..31
                // and rows 64..127 x columns 32..63.
                const uint32_t id = idesc_bf16_f32(128, 64);
#pragma unroll
                for (int pp = 0; pp < 2; ++pp)
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t kb2 = ks >> 2, kin = ks & 3;
                        const uint32_t a = smem_u32(sR) + r_sub(pp, kb2) + kin * 32;
                        const uint32_t b = smem_u32(sKQ) + kb2 * 128 * 128 + 64 * pp * 128 + kin * 32;
                        mma_ss(tmem_addr(tb, 0, 64 * pp), desc_kmajor_sw128(a), desc_kmajor_sw128(b), id, ks > 0);
                    }
                mma_commit(&mma_bar);
            }
            // While the products run, warp 0 requests the next item into the other
            // stage (free: its previous item finished with it).
            if (warp == 0 && w + (int)gridDim.x < total_items) {
                issue(w + gridDim.x, s ^ 1);
                issued = it + 2;
            }
            if (!mbar_wait(&mma_bar, mma_count & 1, globaltimer_ns() + kWaitNs)) {
                if (tid == 0) record_timeout(status);
                sAbort = 1;
                break;
            }
            ++mma_count;
            tc_fence_after_sync();

            float *Af = (float *)(sm + kIAf), *Tf = (float *)(sm + kITf), *Xf = (float *)(sm + kIXf);
            {
                // M = 128 layout: TMEM lane = A row.  Warps 0-7: pair p = warp / 4,
                // lane quarter q = warp % 4; quarters 0-1 hold R^(2p+1) rows (wanted
                // columns 0..31 of the pair), quarters 2-3 hold R^(2p) rows (32..63).
                if (warp < 8) {
                    uint32_t rr[32];
                    const int q = warp & 3, pp = warp >> 2, slot = q >> 1;
                    const int sidx = 32 * (q & 1) + lane, Ia = slot ? 2 * pp : 2 * pp + 1;
                    tmem_ld32(tmem_addr(tb, 32 * q, 64 * pp + 32 * slot), rr);
                    tmem_ld_wait();
#pragma unroll
                    for (int jr = 0; jr < 16; ++jr) {
                        const int r = 16 * Ia + jr;
                        Af[r * kLd + sidx] = sidx < r ? sBeta[s][r] * __uint_as_float(rr[jr]) : 0.f;
                        const float pvv = sidx <= r ? __uint_as_float(rr[16 + jr]) : 0.f;
                        *(__nv_bfloat16 *)(blk + kOffP + sw128_offset(r, sidx, 64)) = __float2bfloat16_rn(pvv);
                    }
                }
            }
            // [beta K e^G ; beta V]^T (256 rows x 64 tokens) into the freed [Kt; Qt] region.
            *(uint4 *)(sKQ + sw128_offset(c0, 8 * q8, 256)) = make_uint4(pk0[0], pk0[1], pk0[2], pk0[3]);
            *(uint4 *)(sKQ + sw128_offset(c0 + 1, 8 * q8, 256)) = make_uint4(pk1[0], pk1[1], pk1[2], pk1[3]);
            *(uint4 *)(sKQ + sw128_offset(128 + c0, 8 * q8, 256)) = make_uint4(pv0[0], pv0[1], pv0[2], pv0[3]);
            *(uint4 *)(sKQ + sw128_offset(128 + c0 + 1, 8 * q8, 256)) = make_uint4(pv1[0], pv1[1], pv1[2], pv1[3]);
            tc_fence_before_sync();
            compute_sync();

            // T, rounded to bf16, is also the A operand of the W/U product
            // (64 rows x 64 K), written into the item's raw k tile as it is formed.
            uint8_t *sT = stw + kRawK;
            // T = (I + A)^-1 by blocks of 16: diagonal blocks by forward
            // substitution, then T_ij = -T_ii A_ij T_jj doubled from 16 to 32 to 64.
            // Only the lower triangle is used; the two upper blocks that the
            // doubling products read, (0,1) and (2,3), are set to zero.
            if (tid < 64) {
                const int Ib = tid >> 4, jc = tid & 15, o = 16 * Ib;
                float col[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    float x = (r == jc) ? 1.f : 0.f;
#pragma unroll
                    for (int s2 = 0; s2 < r; ++s2) x = fmaf(-Af[(o + r) * kLd + o + s2], col[s2], x);
                    col[r] = r < jc ? 0.f : x;
                }
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    Tf[(o + r) * kLd + o + jc] = col[r];
                    *(__nv_bfloat16 *)(sT + sw128_offset(o + r, o + jc, 64)) = __float2bfloat16_rn(col[r]);
                }
            } else {
                const int e = tid - 64;  // the other threads zero the upper blocks
                for (int f = e; f < 512; f += kIntraCompute - 64) {
                    const int blkz = f >> 8, r = (f >> 4) & 15, cz = f & 15;
                    const int ro = 32 * blkz, co = 32 * blkz + 16;
                    Tf[(ro + r) * kLd + co + cz] = 0.f;   // read by the doubling products
                }
                for (int f = e; f < 6 * 256; f += kIntraCompute - 64) {
                    const int bz = f >> 8, r = (f >> 4) & 15, cz = f & 15;
                    // upper blocks (0,1) (0,2) (0,3) (1,2) (1,3) (2,3) of the bf16 operand
                    const int bi = bz < 3 ? 0 : bz < 5 ? 1 : 2;
                    const int bj = bz < 3 ? bz + 1 : bz < 5 ? bz - 1 : 3;
                    *(__nv_bfloat16 *)(sT + sw128_offset(16 * bi + r, 16 * bj + cz, 64)) = __float2bfloat16_rn(0.f);
                }
            }
            compute_sync();
            {
                // Level 1, blocks (1,0) and (3,2): X = A_ij T_jj, one output per thread.
                const int p = tid >> 8, r = (tid >> 4) & 15, sb = tid & 15;
                const int oi = 32 * p + 16, oj = 32 * p;
                float x0 = 0.f, x1 = 0.f;
#pragma unroll
                for (int t = 0; t < 16; t += 2) {
                    x0 = fmaf(Af[(oi + r) * kLd + oj + t], Tf[(oj + t) * kLd + oj + sb], x0);
                    x1 = fmaf(Af[(oi + r) * kLd + oj + t + 1], Tf[(oj + t + 1) * kLd + oj + sb], x1);
                }
                Xf[(16 * p + r) * 33 + sb] = x0 + x1;
                compute_sync();
                float y0 = 0.f, y1 = 0.f;
#pragma unroll
                for (int t = 0; t < 16; t += 2) {
                    y0 = fmaf(Tf[(oi + r) * kLd + oi + t], Xf[(16 * p + t) * 33 + sb], y0);
                    y1 = fmaf(Tf[(oi + r) * kLd + oi + t + 1], Xf[(16 * p + t + 1) * 33 + sb], y1);
                }
                y0 += y1;
                Tf[(oi + r) * kLd + oj + sb] = -y0;
                *(__nv_bfloat16 *)(sT + sw128_offset(oi + r, oj + sb, 64)) = __float2bfloat16_rn(-y0);
            }
            compute_sync();
            {
                // Level 2, block rows 32..63 x columns 0..31: two outputs per thread.
                const int r = tid >> 4, sb = tid & 15;
                float x[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
                for (int t = 0; t < 32; t += 2) {
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const float a = Af[(32 + r) * kLd + t + u];
#pragma unroll
                        for (int jj = 0; jj < 2; ++jj) x[u][jj] = fmaf(a, Tf[(t + u) * kLd + sb + 16 * jj], x[u][jj]);
                    }
                }
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) Xf[r * 33 + sb + 16 * jj] = x[0][jj] + x[1][jj];
                compute_sync();
                float yy[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
                for (int t = 0; t < 32; t += 2) {
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const float tt = Tf[(32 + r) * kLd + 32 + t + u];
#pragma unroll
                        for (int jj = 0; jj < 2; ++jj) yy[u][jj] = fmaf(tt, Xf[(t + u) * 33 + sb + 16 * jj], yy[u][jj]);
                    }
                }
                const float y[2] = {yy[0][0] + yy[1][0], yy[0][1] + yy[1][1]};
#pragma unroll
                for (int jj = 0; jj < 2; ++jj)
                    *(__nv_bfloat16 *)(sT + sw128_offset(32 + r, sb + 16 * jj, 64)) = __float2bfloat16_rn(-y[jj]);
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            compute_sync();
            tc_fence_after_sync();
            if (tid == 0) {
                const uint32_t id = idesc_bf16_f32(64, 256);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_ss(tmem_addr(tb, 0, 0), desc_kmajor_sw128(smem_u32(sT) + ks * 32),
                           desc_kmajor_sw128(smem_u32(sKQ) + ks * 32), id, ks > 0);
                mma_commit(&mma_bar);
            }
            if (!mbar_wait(&mma_bar, mma_count & 1, globaltimer_ns() + kWaitNs)) {
                if (tid == 0) record_timeout(status);
                sAbort = 1;
                break;
            }
            ++mma_count;
            tc_fence_after_sync();
            {
                // W (columns 0..127) -> rows 0..63 of [W; Qt]; U (columns 128..255).
                // Warp w: lane quadrant w % 4, columns 64 (w / 4) .. + 63.
                uint32_t rr[32];
                const int wq = warp & 3, r = 16 * wq + lane, cg = warp >> 2;
                uint32_t rr2[32];
                tmem_ld32(tmem_addr(tb, 32 * wq, 64 * cg), rr);
                tmem_ld32(tmem_addr(tb, 32 * wq, 64 * cg + 32), rr2);
                tmem_ld_wait();
#pragma unroll
                for (int q4 = 0; q4 < 2; ++q4) {
                    const int colbase = 64 * cg + 32 * q4;
                    if (q4 == 1) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) rr[i] = rr2[i];
                    }
                    if (lane < 16) {
#pragma unroll
                        for (int cc = 0; cc < 32; cc += 8) {
                            const uint4 w4 = make_uint4(
                                pack_bf16(__uint_as_float(rr[cc]), __uint_as_float(rr[cc + 1])),
                                pack_bf16(__uint_as_float(rr[cc + 2]), __uint_as_float(rr[cc + 3])),
                                pack_bf16(__uint_as_float(rr[cc + 4]), __uint_as_float(rr[cc + 5])),
                                pack_bf16(__uint_as_float(rr[cc + 6]), __uint_as_float(rr[cc + 7])));
                            const int col = colbase + cc;
                            // Staged as block images: W (two 64-wide K halves of rows
                            // 0..63 of [W; Qt]) in the v tile, U (row-major) in the q tile.
                            if (col < 128)
                                *(uint4 *)(stw + kRawV + (col >> 6) * 8192 + sw128_offset(r, col & 63, 64)) = w4;
                            else
                                *(uint4 *)(stw + kRawQ + (r * 128 + col - 128) * 2) = w4;
                        }
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            compute_sync();
            if (tid == 0) {
                bulk_s2g(blk + kOffWQ, stw + kRawV, 8192);
                bulk_s2g(blk + kOffWQ + 16384, stw + kRawV + 8192, 8192);
                bulk_s2g(blk + kOffU, stw + kRawQ, 16384);
                bulk_commit();
            }
        }
        if (tid == 0) bulk_wait<0>();  // every staged block region has reached memory
        // Drain: every requested copy has landed before the CTA may exit.
        if (warp == 0) {
            cp_async_wait_all();
            for (int d = it; d < issued; ++d)
                mbar_wait(&full[d & 1], (d >> 1) & 1, globaltimer_ns() + kWaitNs);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, 256);
}

// ------------------------------------------------------------------ state --

constexpr int kStateThreads = 320;       // epilogue: warps 0-7, load: 8, mma: 9
constexpr uint32_t kStageBytes = 75776;  // block rounded up to 1 KiB
constexpr int kStages = 2;
constexpr uint32_t kOStage = kStages * kStageBytes;  // 2 x [64][128] bf16 output staging
constexpr uint32_t kStateSmem = kStages * kStageBytes + 2 * 16384 + 1024;
// TMEM columns
constexpr uint32_t kTS = 0, kTSbf = 128, kTDl = 192, kTD1 = 256;  // D1 double buffer: 256, 384

struct StateBars {
    uint64_t full[kStages], empty[kStages];
    uint64_t mma1, dl_ready, sbf_ready, sdec_ready;
    uint64_t mma2[2], d1_free[2], ostaged[2];
};
constexpr uint32_t kEpi = 256;  // epilogue threads: two warpgroups

// Segments: with G > 1 every sequence of nch chunks is cut into Gn = min(G, nch)
// runs of chunks, [s nch / Gn, (s + 1) nch / Gn), and each (sequence, head) gets
// 2 G - 1 CTAs ("slots"):
//   slot 0          segment 0 from the true initial state; outputs -> o;
//   slot 2 s - 1    segment s from a zero state (S_loc); outputs -> o (partial);
//   slot 2 s        segment s on the transition X, X_0 = I and U = 0; its state
//                   after the segment is the dk x dk map M_s, its outputs are
//                   E = (Qt - P W) X per chunk, written as MMA A-operand images.
// Segment ends: slot 0 -> Sx[n][0][h], slot 2s-1 -> Sx[n][s][h], slot 2s ->
// Mx[n][s][h]; compose_kernel and correct_kernel finish the job.  With G == 1
// the single slot writes the final state and checkpoints directly.
__device__ __forceinline__ int seg_begin(int s, int nch, int Gn) {
    return (int)(((int64_t)s * nch) / Gn);
}
constexpr uint32_t kEImg = kChunk * kDK * 2;    // E image of one (chunk, head): 16 KiB
constexpr uint32_t kSinImg = kDV * kDK * 2;     // S_in image of one (segment, head): 32 KiB
constexpr size_t kStateF32 = (size_t)kDK * kDV;  // one fp32 state, in floats

__global__ void __launch_bounds__(kStateThreads, 1)
state_kernel(const int32_t *__restrict__ cu, const int32_t *__restrict__ chunk_off,
             const int32_t *__restrict__ order, int N, int H,
             const uint8_t *__restrict__ blocks, int64_t max_chunks,
             const float *S0user, float *Sfuser, __nv_bfloat16 *__restrict__ o, int32_t *status,
             int ckpt_every, const int32_t *__restrict__ ckpt_off, float *__restrict__ ckpts,
             int G, float *__restrict__ Sx, float *__restrict__ Mx, uint8_t *__restrict__ Eimg)
{
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
    __shared__ StateBars bars;
    __shared__ uint32_t tbase;
    __shared__ volatile int sAbort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slots = 2 * G - 1;
    const int slot = blockIdx.x % slots;
    const int n = order[(blockIdx.x / slots) / H], h = (blockIdx.x / slots) % H;
    const int nch_seq = chunk_off[n + 1] - chunk_off[n];
    const int Gn = min(G, nch_seq);
    const size_t sbase = ((size_t)n * H + h) * kDK * kDV;

    if (nch_seq == 0) {  // empty sequence: the state passes through
        if (Sfuser && slot == 0)
            for (int e = tid; e < kDK * kDV; e += kStateThreads)
                Sfuser[sbase + e] = S0user ? S0user[sbase + e] : 0.f;
        return;
    }
    if (slot >= 2 * Gn - 1) return;  // a segment this short sequence does not have
    const int seg = (slot + 1) >> 1;
    const bool xmode = slot > 0 && (slot & 1) == 0;  // transition X of segment seg
    const int cbeg = seg_begin(seg, nch_seq, Gn);
    const int nch = seg_begin(seg + 1, nch_seq, Gn) - cbeg;
    const int tbeg = cu[n] + cbeg * kChunk, tend = cu[n + 1];
    const float *S0 = slot == 0 ? S0user : nullptr;
    const size_t xbase = (((size_t)n * G + seg) * H + h) * kStateF32;
    float *Sf = Gn == 1 ? Sfuser : (xmode ? Mx + xbase : Sx + xbase);
    const size_t fbase = Gn == 1 ? sbase : 0;  // Sf offset of this (sequence, head)
    uint8_t *eimg = xmode ? Eimg + ((size_t)h * max_chunks + chunk_off[n] + cbeg) * kEImg : nullptr;
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) { mbar_init(&bars.full[s], 1); mbar_init(&bars.empty[s], kEpi + 1); }
        mbar_init(&bars.mma1, 1);
        mbar_init(&bars.dl_ready, kEpi);
        mbar_init(&bars.sbf_ready, kEpi);
        mbar_init(&bars.sdec_ready, kEpi);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars.mma2[b], 1);
            mbar_init(&bars.d1_free[b], kEpi);
            mbar_init(&bars.ostaged[b], kEpi);
        }
        fence_mbar_init();
        sAbort = 0;
    }
    if (warp == 0) { tmem_alloc(&tbase, 512); tmem_relinquish(); }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tb = tbase;
    const uint8_t *blk0 = blocks + ((size_t)h * max_chunks + chunk_off[n] + cbeg) * kBlockBytes;

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
                if (!mbar_wait(&bars.dl_ready, c & 1, globaltimer_ns() + kWaitNs) ||
                    !mbar_wait(&bars.sdec_ready, c & 1, globaltimer_ns() + kWaitNs)) {
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
    } else {
        // ---- epilogue, warps 0-7: thread j = TMEM lane = value channel j; half hh
        // takes delta rows 32 hh .., state columns 64 hh .. and output rows 32 hh .. ----
        const int j = tid & 127, hh = warp >> 2;
        const uint32_t lq = 32 * (warp & 3);
        uint32_t ra[32], rb[32];
        // Initial state: S^T row j = column j of S0 (this half's 64 key channels):
        // fp32 master pre-multiplied by the first chunk's decay, and the bf16 copy.
        // The transition X starts from the identity: X^T row j = e_j.
        bool ok = true;
        const float *dec0 = nullptr;
        const bool nonzero0 = S0 || xmode;
        if (nonzero0) {
            ok = mbar_wait(&bars.full[0], 0, globaltimer_ns() + kWaitNs);
            if (!ok) { record_timeout(status); sAbort = 1; }
            dec0 = (const float *)(sm + kOffDecay);
        }
        for (int q2 = 0; q2 < 2 && ok; ++q2) {
            const int c0 = 64 * hh + 32 * q2;
            float sv[32];
#pragma unroll
            for (int i = 0; i < 32; ++i)
                sv[i] = S0 ? S0[sbase + (size_t)(c0 + i) * kDV + j] : (xmode && c0 + i == j ? 1.f : 0.f);
#pragma unroll
            for (int i = 0; i < 32; ++i) ra[i] = __float_as_uint(nonzero0 ? sv[i] * dec0[c0 + i] : 0.f);
            tmem_st32(tmem_addr(tb, lq, kTS + c0), ra);
            uint32_t sb[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) sb[i] = pack_bf16(sv[2 * i], sv[2 * i + 1]);
            tmem_st16(tmem_addr(tb, lq, kTSbf + c0 / 2), sb);
        }
        tmem_st_wait();
        tc_fence_before_sync();
        mbar_arrive(&bars.sbf_ready);
        mbar_arrive(&bars.sdec_ready);

        // O^T rows of chunk cc -> o: each thread parks its 32 values in a [64][128]
        // bf16 staging tile (double-buffered by chunk parity), then the 256
        // threads write whole 256-byte token rows with 16-byte stores.
        auto output = [&](int cc) {
            const int bb = cc & 1;
            const int t0 = tbeg + cc * kChunk;
            const int len = min(kChunk, tend - t0);
            __nv_bfloat16 *ost = (__nv_bfloat16 *)(sm + kOStage + bb * 16384);
            tmem_ld32(tmem_addr(tb, lq, kTD1 + 128 * bb + 64 + 32 * hh), ra);
            tmem_ld_wait();
            tc_fence_before_sync();
            mbar_arrive(&bars.d1_free[bb]);
#pragma unroll
            for (int i = 0; i < 32; ++i) ost[(32 * hh + i) * kDV + j] = __float2bfloat16_rn(__uint_as_float(ra[i]));
            mbar_arrive(&bars.ostaged[bb]);
            if (!mbar_wait(&bars.ostaged[bb], (cc >> 1) & 1, globaltimer_ns() + kWaitNs)) {
                record_timeout(status);
                sAbort = 1;
                return;
            }
            const int r = tid >> 2, part = tid & 3;
            const uint4 *src = (const uint4 *)(ost + r * kDV + 32 * part);
            if (eimg) {
                // E rows as the K-major, 128-byte-swizzled A operand of the
                // correction product (two 64-wide K halves of 64 rows each).
                uint8_t *dst = eimg + (size_t)cc * kEImg;
#pragma unroll
                for (int m = 0; m < 4; ++m)
                    *(uint4 *)(dst + ((32 * part + 8 * m) >> 6) * 8192 +
                               sw128_offset(r, (32 * part + 8 * m) & 63, 64)) = src[m];
            } else if (r < len) {
                uint4 *dst = (uint4 *)(o + ((size_t)(t0 + r) * H + h) * kDV + 32 * part);
#pragma unroll
                for (int m = 0; m < 4; ++m) dst[m] = src[m];
            }
        };

        for (int c = 0; c < nch && !sAbort; ++c) {
            const int s = c % kStages, b = c & 1;
            const uint8_t *st = sm + s * kStageBytes;
            if (!mbar_wait(&bars.full[s], (c / kStages) & 1, globaltimer_ns() + kWaitNs) ||
                !mbar_wait(&bars.mma1, c & 1, globaltimer_ns() + kWaitNs)) {
                record_timeout(status); sAbort = 1; break;
            }
            tc_fence_after_sync();
            // Dl^T[j][r] = U[r][j] - D1[j][r] for this half's 32 rows -> bf16 pairs into TMEM
            // (U = 0 on the transition).
            {
                const __nv_bfloat16 *U = (const __nv_bfloat16 *)(st + kOffU);
                tmem_ld32(tmem_addr(tb, lq, kTD1 + 128 * b + 32 * hh), ra);
                tmem_ld_wait();
                uint32_t dl[16];
                if (xmode) {
#pragma unroll
                    for (int i = 0; i < 32; i += 2)
                        dl[i >> 1] = pack_bf16(-__uint_as_float(ra[i]), -__uint_as_float(ra[i + 1]));
                } else {
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        const int r = 32 * hh + i;
                        const float d0 = __bfloat162float(U[r * kDV + j]) - __uint_as_float(ra[i]);
                        const float d1v = __bfloat162float(U[(r + 1) * kDV + j]) - __uint_as_float(ra[i + 1]);
                        dl[i >> 1] = pack_bf16(d0, d1v);
                    }
                }
                tmem_st16(tmem_addr(tb, lq, kTDl + 16 * hh), dl);
                tmem_st_wait();
            }
            tc_fence_before_sync();
            mbar_arrive(&bars.dl_ready);
            mbar_arrive(&bars.empty[s]);  // done with U of this stage
            // The previous chunk's output, off the critical path (its D1 buffer is
            // only reused by the product two chunks later).
            if (c > 0) output(c - 1);

            if (!mbar_wait(&bars.mma2[b], (c >> 1) & 1, globaltimer_ns() + kWaitNs)) {
                record_timeout(status); sAbort = 1; break;
            }
            tc_fence_after_sync();
            const bool last = (c + 1 == nch);
            // S_out, this half's 64 key channels: two loads, one wait.
            tmem_ld32(tmem_addr(tb, lq, kTS + 64 * hh), ra);
            tmem_ld32(tmem_addr(tb, lq, kTS + 64 * hh + 32), rb);
            tmem_ld_wait();
            // Checkpoint when the state after `pos` tokens falls on a multiple of every.
            const int pos = min((c + 1) * kChunk, tend - tbeg);
            if (ckpt_every > 0 && pos % ckpt_every == 0) {
                float *ck = ckpts + ((size_t)(ckpt_off[n] + pos / ckpt_every - 1) * H + h) * kDK * kDV;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    ck[(size_t)(64 * hh + i) * kDV + j] = __uint_as_float(ra[i]);
                    ck[(size_t)(64 * hh + 32 + i) * kDV + j] = __uint_as_float(rb[i]);
                }
            }
            if (last) {
                if (Sf) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        Sf[fbase + (size_t)(64 * hh + i) * kDV + j] = __uint_as_float(ra[i]);
                        Sf[fbase + (size_t)(64 * hh + 32 + i) * kDV + j] = __uint_as_float(rb[i]);
                    }
                }
            } else {
                // Critical: the bf16 copy that the next chunk's first product reads.
                uint32_t sa[16], sbv[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    sa[i] = pack_bf16(__uint_as_float(ra[2 * i]), __uint_as_float(ra[2 * i + 1]));
                    sbv[i] = pack_bf16(__uint_as_float(rb[2 * i]), __uint_as_float(rb[2 * i + 1]));
                }
                tmem_st16(tmem_addr(tb, lq, kTSbf + 32 * hh), sa);
                tmem_st16(tmem_addr(tb, lq, kTSbf + 32 * hh + 16), sbv);
                tmem_st_wait();
                tc_fence_before_sync();
                mbar_arrive(&bars.sbf_ready);
                // Off the critical path: the fp32 master times the next chunk's decay.
                const int s1 = (c + 1) % kStages;
                if (!mbar_wait(&bars.full[s1], ((c + 1) / kStages) & 1, globaltimer_ns() + kWaitNs)) {
                    record_timeout(status); sAbort = 1; break;
                }
                const float *dec = (const float *)(sm + s1 * kStageBytes + kOffDecay) + 64 * hh;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    ra[i] = __float_as_uint(__uint_as_float(ra[i]) * dec[i]);
                    rb[i] = __float_as_uint(__uint_as_float(rb[i]) * dec[32 + i]);
                }
                tmem_st32(tmem_addr(tb, lq, kTS + 64 * hh), ra);
                tmem_st32(tmem_addr(tb, lq, kTS + 64 * hh + 32), rb);
                tmem_st_wait();
                tc_fence_before_sync();
                mbar_arrive(&bars.sdec_ready);
            }
        }
        if (!sAbort) output(nch - 1);  // the last chunk's output
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, 512);
}

// ---------------------------------------------------------------- compose --

// Affine composition of the segments of one (sequence, head), for 32 value
// channels per CTA (columns of S never mix):
//   S_in(1) = S after segment 0,   S_in(s + 1) = M_s S_in(s) + S_loc(s),
// the final state being S_in(Gn).  The whole scan is in fp32; each S_in(s) is
// also written as the bf16 B-operand image (row = value channel, K = key
// channel, 128-byte swizzled) that the correction product reads.
constexpr int kComposeThreads = 256;
constexpr int kComposeCols = 32;
constexpr int kMsLd = kDK + 1;
constexpr uint32_t kComposeSmem = (kDK * kMsLd + kDK * kComposeCols) * 4;

__global__ void __launch_bounds__(kComposeThreads)
compose_kernel(const int32_t *__restrict__ chunk_off, int H, int G, const float *__restrict__ Sx,
               const float *__restrict__ Mx, uint8_t *__restrict__ Simg, float *Sf)
{
    extern __shared__ float csm[];
    float *Ms = csm;                 // M_s [128][129]
    float *Ss = csm + kDK * kMsLd;   // S_in(s), this CTA's columns [128][32]
    constexpr int nvb = kDV / kComposeCols;
    const int vb = blockIdx.x % nvb, h = (blockIdx.x / nvb) % H, n = blockIdx.x / (nvb * H);
    const int Gn = min(G, chunk_off[n + 1] - chunk_off[n]);
    if (Gn <= 1) return;             // the state kernel wrote this final state itself
    const int tid = threadIdx.x;
    const int m = tid >> 1, cb = (tid & 1) * 16, v0 = vb * kComposeCols;
    auto xoff = [&](int s) { return (((size_t)n * G + s) * H + h) * kStateF32; };

    for (int e = tid; e < kDK * kComposeCols; e += kComposeThreads)
        Ss[e] = Sx[xoff(0) + (size_t)(e / kComposeCols) * kDV + v0 + e % kComposeCols];
    __syncthreads();
    for (int s = 1; s < Gn; ++s) {
        uint8_t *img = Simg + (((size_t)n * G + s) * H + h) * kSinImg;
#pragma unroll
        for (int i = 0; i < 16; ++i)
            *(__nv_bfloat16 *)(img + sw128_offset(v0 + cb + i, m, kDV)) =
                __float2bfloat16_rn(Ss[m * kComposeCols + cb + i]);
        const float4 *Mg = (const float4 *)(Mx + xoff(s));
        for (int e = tid; e < kDK * kDK / 4; e += kComposeThreads) {
            const float4 x = Mg[e];
            float *d = Ms + (e >> 5) * kMsLd + 4 * (e & 31);
            d[0] = x.x; d[1] = x.y; d[2] = x.z; d[3] = x.w;
        }
        __syncthreads();
        float acc[16];
        const float *Sl = Sx + xoff(s) + (size_t)m * kDV + v0 + cb;
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = Sl[i];
        for (int c = 0; c < kDK; ++c) {
            const float a = Ms[m * kMsLd + c];
            const float4 *sr = (const float4 *)(Ss + c * kComposeCols + cb);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 x = sr[q];
                acc[4 * q + 0] = fmaf(a, x.x, acc[4 * q + 0]);
                acc[4 * q + 1] = fmaf(a, x.y, acc[4 * q + 1]);
                acc[4 * q + 2] = fmaf(a, x.z, acc[4 * q + 2]);
                acc[4 * q + 3] = fmaf(a, x.w, acc[4 * q + 3]);
            }
        }
        __syncthreads();             // every read of Ss and Ms is done
#pragma unroll
        for (int i = 0; i < 16; ++i) Ss[m * kComposeCols + cb + i] = acc[i];
        __syncthreads();
    }
    if (Sf) {
        float *d = Sf + ((size_t)n * H + h) * kStateF32 + (size_t)m * kDV + v0 + cb;
#pragma unroll
        for (int i = 0; i < 16; ++i) d[i] = Ss[m * kComposeCols + cb + i];
    }
}

// ---------------------------------------------------------------- correct --

// Outputs of a chunk in segment s >= 1: o += E S_in(s), one tcgen05 product
// (M = 64 tokens, N = 128 value channels, K = 128 key channels) per
// (chunk, head), fp32 in TMEM, added to the bf16 partial output in place.
constexpr int kCorrThreads = 128;
constexpr uint32_t kCorrSmem = kEImg + kSinImg + 1024;

__global__ void __launch_bounds__(kCorrThreads)
correct_kernel(const int32_t *__restrict__ cu, const int32_t *__restrict__ chunk_off, int N, int H,
               int G, int64_t max_chunks, const uint8_t *__restrict__ Eimg,
               const uint8_t *__restrict__ Simg, __nv_bfloat16 *__restrict__ o, int32_t *status)
{
    const int h = blockIdx.x % H;
    const int g = blockIdx.x / H;    // global chunk index
    if (g >= chunk_off[N]) return;
    const int n = find_seq(chunk_off, N, g);
    const int nch = chunk_off[n + 1] - chunk_off[n];
    const int Gn = min(G, nch), c = g - chunk_off[n];
    if (Gn <= 1) return;
    int s = 0;
    while (s + 1 < Gn && seg_begin(s + 1, nch, Gn) <= c) ++s;
    if (s == 0) return;              // segment 0 started from the true state

    extern __shared__ uint8_t smraw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smraw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t bar_ld, bar_mma;
    __shared__ uint32_t tbase;
    __shared__ int sOk;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        mbar_init(&bar_ld, 1);
        mbar_init(&bar_mma, 1);
        fence_mbar_init();
        sOk = 0;
    }
    if (warp == 0) { tmem_alloc(&tbase, 128); tmem_relinquish(); }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tb = tbase;
    if (tid == 0) {
        mbar_arrive_expect_tx(&bar_ld, kEImg + kSinImg);
        bulk_g2s(sm, Eimg + ((size_t)h * max_chunks + g) * kEImg, kEImg, &bar_ld);
        bulk_g2s(sm + kEImg, Simg + (((size_t)n * G + s) * H + h) * kSinImg, kSinImg, &bar_ld);
        if (mbar_wait(&bar_ld, 0, globaltimer_ns() + kWaitNs)) {
            tc_fence_after_sync();
            const uint32_t id = idesc_bf16_f32(64, 128), ea = smem_u32(sm), sa = smem_u32(sm + kEImg);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_ss(tmem_addr(tb, 0, 0), desc_kmajor_sw128(ea + (ks >> 2) * 8192 + (ks & 3) * 32),
                       desc_kmajor_sw128(sa + (ks >> 2) * 16384 + (ks & 3) * 32), id, ks > 0);
            mma_commit(&bar_mma);
            sOk = mbar_wait(&bar_mma, 0, globaltimer_ns() + kWaitNs) ? 1 : 0;
        } else {
            // Drain: the copies must land before the CTA's shared memory is released.
            mbar_wait(&bar_ld, 0, globaltimer_ns() + kWaitNs);
        }
        if (!sOk) record_timeout(status);
    }
    __syncthreads();
    if (sOk) {
        tc_fence_after_sync();
        const int t0 = cu[n] + c * kChunk, len = min(kChunk, cu[n + 1] - t0);
        const int r = 16 * warp + lane;  // M = 64: TMEM lane 32 w + i holds row 16 w + i
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
            uint32_t ra[32];
            tmem_ld32(tmem_addr(tb, 32 * warp, 32 * q), ra);
            tmem_ld_wait();
            if (lane < 16 && r < len) {
                uint4 *d4 = (uint4 *)(o + ((size_t)(t0 + r) * H + h) * kDV + 32 * q);
#pragma unroll
                for (int m4 = 0; m4 < 4; ++m4) {
                    uint4 x = d4[m4];
                    uint32_t *w = &x.x;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(*(const __nv_bfloat162 *)&w[e]);
                        w[e] = pack_bf16(f.x + __uint_as_float(ra[8 * m4 + 2 * e]),
                                         f.y + __uint_as_float(ra[8 * m4 + 2 * e + 1]));
                    }
                    d4[m4] = x;
                }
            }
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, 128);
}

// cuTensorMapEncodeTiled, fetched from the driver through the runtime (no
// link-time dependency on libcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
    });
    return fn;
}

// [T][H][128] bf16 rows viewed as a 3-D tensor (channel, head, token) with a
// {128, 1, 64} box: one chunk of one head per load, no swizzle.
bool encode_rows_map(CUtensorMap *map, const void *base, int32_t T, int32_t H)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)kDK, (cuuint64_t)H, (cuuint64_t)(T > 0 ? T : 1)};
    const cuuint64_t strides[2] = {(cuuint64_t)kDK * 2, (cuuint64_t)H * kDK * 2};
    const cuuint32_t box[3] = {(cuuint32_t)kDK, 1, (cuuint32_t)kChunk};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

namespace {

// SMs the split plan targets: the 148 of a B200.
constexpr int64_t kSplitSms = 148;
constexpr int64_t kMaxSegments = 16;

// Workspace layout: plan region, per-(chunk, head) blocks, then (split only)
// Sx and Mx [N][G][H] fp32 states, S_in images [N][G][H] and E images [H][chunks].
struct WsLayout {
    size_t plan, blocks, sx, mx, simg, eimg, total;
};

WsLayout ws_layout(int32_t total_tokens, int32_t num_seqs, int32_t H, int G)
{
    WsLayout w{};
    if (num_seqs <= 0) return w;
    const int64_t max_chunks = ((int64_t)total_tokens + 63LL * num_seqs) / kChunk;
    auto up = [](size_t x) { return (x + 1023) & ~(size_t)1023; };
    w.plan = 0;
    w.blocks = up((size_t)(3 * num_seqs + 3) * sizeof(int32_t));
    size_t end = w.blocks + (size_t)H * max_chunks * kBlockBytes;
    if (G > 1) {
        const size_t states = (size_t)num_seqs * G * H;
        w.sx = up(end);
        w.mx = w.sx + states * kStateF32 * sizeof(float);
        w.simg = w.mx + states * kStateF32 * sizeof(float);
        w.eimg = w.simg + states * kSinImg;
        end = w.eimg + (size_t)H * max_chunks * kEImg;
    }
    w.total = end;
    return w;
}

}  // namespace

int tc_split_segments(int32_t total_tokens, int32_t num_seqs, int32_t H, bool forced)
{
    if (num_seqs <= 0 || H <= 0) return 1;
    const int64_t chains = (int64_t)num_seqs * H;
    // 2 G - 1 CTAs per (sequence, head) should fit on the SMs at once.
    int64_t G = (kSplitSms / chains + 1) / 2;
    if (G > kMaxSegments) G = kMaxSegments;
    if (!forced) {
        // Only worth it when every segment keeps at least 16 chunks on average.
        const int64_t avg_chunks = (int64_t)total_tokens / ((int64_t)kChunk * num_seqs);
        if (G > avg_chunks / 16) G = avg_chunks / 16;
    } else if (G < 2) {
        G = 2;
    }
    return G < 2 ? 1 : (int)G;
}

size_t tc_workspace_bytes(int32_t total_tokens, int32_t num_seqs, int32_t H, int segments)
{
    return ws_layout(total_tokens, num_seqs, H, segments).total;
}

cudaError_t launch_prefill_tensor_core(const PrefillArgs &a, cudaStream_t stream)
{
    if (a.dk != kDK || a.dv != kDV || !a.bf16) return cudaErrorInvalidValue;
    const int G = a.segments > 1 ? a.segments : 1;
    if (G > 1 && a.ckpt_every > 0) return cudaErrorInvalidValue;
    const int64_t max_chunks = ((int64_t)a.total_tokens + 63LL * a.num_seqs) / kChunk;
    const WsLayout w = ws_layout(a.total_tokens, a.num_seqs, a.H, G);
    uint8_t *ws = (uint8_t *)a.workspace;
    int32_t *chunk_off = (int32_t *)ws;
    int32_t *ckpt_off = chunk_off + a.num_seqs + 1;
    int32_t *order = ckpt_off + a.num_seqs + 1;
    uint8_t *blocks = ws + w.blocks;
    float *Sx = G > 1 ? (float *)(ws + w.sx) : nullptr;
    float *Mx = G > 1 ? (float *)(ws + w.mx) : nullptr;
    uint8_t *Simg = G > 1 ? ws + w.simg : nullptr;
    uint8_t *Eimg = G > 1 ? ws + w.eimg : nullptr;
    cudaError_t err;

    err = cudaFuncSetAttribute(intra_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)(kISmem + 1024));
    if (err != cudaSuccess) return err;
    err = cudaFuncSetAttribute(state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kStateSmem);
    if (err != cudaSuccess) return err;
    if (G > 1) {
        err = cudaFuncSetAttribute(compose_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)kComposeSmem);
        if (err != cudaSuccess) return err;
        err = cudaFuncSetAttribute(correct_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)kCorrSmem);
        if (err != cudaSuccess) return err;
    }

    a.mark(0, stream);
    plan_kernel<<<1, kPlanThreads, 0, stream>>>(a.cu_seqlens, a.num_seqs, a.ckpt_every, chunk_off,
                                                ckpt_off, order);
    a.mark(1, stream);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;

    if (max_chunks > 0) {
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) == cudaSuccess)
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const int64_t items = max_chunks * a.H;
        const unsigned grid = (unsigned)(items < sms ? items : sms);
        CUtensorMap mk, mq, mv, mz;
        if (!encode_rows_map(&mk, a.k, a.total_tokens, a.H) || !encode_rows_map(&mq, a.q, a.total_tokens, a.H) ||
            !encode_rows_map(&mv, a.v, a.total_tokens, a.H) || !encode_rows_map(&mz, a.z, a.total_tokens, a.H))
            return cudaErrorInvalidValue;
        intra_kernel<<<grid, kIntraThreads, kISmem + 1024, stream>>>(
            mk, mq, mv, mz, a.A, a.beta, a.cu_seqlens, chunk_off, a.num_seqs, a.H,
            blocks, max_chunks, a.status);
        err = cudaGetLastError();
        if (err != cudaSuccess) return err;
    }
    a.mark(2, stream);
    state_kernel<<<(unsigned)((int64_t)a.num_seqs * a.H * (2 * G - 1)), kStateThreads, kStateSmem,
                   stream>>>(
        a.cu_seqlens, chunk_off, order, a.num_seqs, a.H, blocks, max_chunks, a.initial_state,
        a.final_state, (__nv_bfloat16 *)a.o, a.status, a.ckpt_every, ckpt_off, a.checkpoints,
        G, Sx, Mx, Eimg);
    a.mark(3, stream);
    err = cudaGetLastError();
    if (err != cudaSuccess || G == 1) return err;

    compose_kernel<<<(unsigned)((int64_t)a.num_seqs * a.H * (kDV / kComposeCols)), kComposeThreads,
                     kComposeSmem, stream>>>(chunk_off, a.H, G, Sx, Mx, Simg, a.final_state);
    a.mark(4, stream);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    if (max_chunks > 0)
        correct_kernel<<<(unsigned)(max_chunks * a.H), kCorrThreads, kCorrSmem, stream>>>(
            a.cu_seqlens, chunk_off, a.num_seqs, a.H, G, max_chunks, Eimg, Simg,
            (__nv_bfloat16 *)a.o, a.status);
    a.mark(5, stream);
    return cudaGetLastError();
}

}  // namespace kda
