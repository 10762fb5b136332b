// Chunked KDA prefill on tcgen05 tensor cores (bf16 operands, fp32 accumulate).
//
// Source: "Kimi K3: Architecture, Training, and Million-Token Agentic RL",
// section 3.1 (recurrence), 3.2 (edit order) and 3.3 (chunked prefill: tokens
// of a chunk become matrix products and the state crosses only chunk
// boundaries; the lower-bounded gate keeps a 16-token tile's cumulative
// log-decay in (-80, 0), so the reciprocal factors stay below e^80 and the
// diagonal tiles use the same dense matrix multiply as the off-diagonal ones).
//
// Three launches per call (five when sequences are split into segments):
//   1. plan:   per-sequence chunk offsets, a per-chunk (first token, length)
//              table and a longest-first order.
//   2. intra:  persistent, two CTAs of 256 threads per SM over the (64-token
//              chunk, head) items.  Gate and cumulative log-decay G in fp32, then
//              on the tensor cores
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
//   4. compose and 5. correct (sequence split only): the affine scan over a
//              sequence's segments and the output correction o += E S_in.
//   (kda_prefill_debug adds a stand-alone gate kernel and a block unpacker.)
//
// Within a chunk (tokens r, s; G inclusive from the chunk start):
//   Dl = (I + A)^-1 Diag(beta) (V - Kt S_in) = U - W S_in,
//   O  = Qt S_in + P Dl,   S_out = Diag(e^{G_C}) S_in + Kd^T Dl,
// the recurrence unrolled over the chunk (the derivation is restated in the
// oracle's chunkwise module).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cstring>
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
constexpr uint32_t kOffKd = 32768;     // Kd^T 128 rows (key channel) x 64 K (token), no swizzle (kd_offset)
constexpr uint32_t kOffP = 49152;      // P 64 rows x 64 K
constexpr uint32_t kOffU = 57344;      // U [64][128] bf16 in 16-channel blocks (u_offset)
constexpr uint32_t kOffDecay = 73984;  // e^{G_C} [128] fp32
constexpr uint32_t kBlockBytes = 74496;
// U element (r, j): blocks of 16 channels, 32 B per row within a block, blocks
// 2080 B apart.  Each store of the intra kernel's readback (16 rows x 16
// channels) then fills 512 contiguous bytes instead of 16 separate 32-byte
// pieces, and the 32-byte skew between blocks (2080 = 16 x 128 + 32) puts the
// two blocks that a state-kernel warp reads for one row (32 channels) on
// different shared-memory banks.
constexpr uint32_t kUBlock = 2080;
__host__ __device__ __forceinline__ uint32_t u_offset(uint32_t r, uint32_t j) {
    return (j >> 4) * kUBlock + r * 32u + (j & 15u) * 2u;
}
// Kd^T element (channel c, token t): K-major without swizzle, 8-channel x
// 16-byte core matrices (channels 16 B apart, SBO = 128 B), 8-token groups
// 2048 B apart (LBO).  A warp's store of 32 channels x 8 tokens then covers 8
// lines instead of 32.
constexpr uint32_t kKdLbo = 2048, kKdSbo = 128;
__host__ __device__ __forceinline__ uint32_t kd_offset(uint32_t c, uint32_t t) {
    return (t >> 3) * kKdLbo + c * 16u + (t & 7u) * 2u;
}

// The dynamic shared memory rounded up to a 1024-byte boundary (the 128-byte
// swizzle's period).  The offset is added to the __shared__ pointer itself, not
// through an integer round trip, so the compiler still knows every access made
// through the result is a shared-memory access (32-bit addressing, LDS/STS).
__device__ __forceinline__ uint8_t *align_smem_1024(uint8_t *smraw) {
    return smraw + ((1024u - (smem_u32(smraw) & 1023u)) & 1023u);
}

__device__ __forceinline__ void record_timeout(int32_t *status) {
    atomicCAS(status, 0, (int32_t)KDA_TC_TIMEOUT_CODE);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&p);
}


// ------------------------------------------------------------------- plan --

__device__ __forceinline__ int find_seq(const int32_t *chunk_off, int N, int g) {
    int lo = 0, hi = N - 1;  // largest n with chunk_off[n] <= g
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (chunk_off[mid] <= g) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// chunk_off[n] = sum_{m<n} ceil(L_m / 64); chunk_off[N] = total chunks.
// ckpt_off[n] = sum_{m<n} L_m / every (checkpoint rows), when every > 0.
// order[i] = sequence index with the i-th largest length (ties by index)
// when N <= kMaxSorted, else the identity.
// chunk_loc[g] = (first token, length) of global chunk g.
constexpr int kPlanThreads = 1024;
constexpr int kMaxSorted = 4096;

__global__ void __launch_bounds__(kPlanThreads)
plan_kernel(const int32_t *__restrict__ cu, int N, int every, int32_t *__restrict__ chunk_off,
            int32_t *__restrict__ ckpt_off, int32_t *__restrict__ order, int2 *__restrict__ chunk_loc)
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
    __syncthreads();  // chunk_off is complete
    const int total = part[0][kPlanThreads - 1];
    for (int g = tid; g < total; g += kPlanThreads) {
        const int n = find_seq(chunk_off, N, g);
        const int t0 = cu[n] + (g - chunk_off[n]) * kChunk;
        chunk_loc[g] = make_int2(t0, min(kChunk, cu[n + 1] - t0));
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

// Persistent, two CTAs of 256 threads per SM, each walking (chunk, head) items
// b, b + gridDim.x, ...; item w is chunk w / H of head w % H.  A CTA holds one
// item at a time; the SM's other CTA overlaps its waits (loads, products,
// barriers).  Thread (cp, p) owns channels 2 cp, 2 cp + 1 of the 8-row
// half-blocks p and 7 - p (p = warp / 2), so the rows' sub-tiles are uniform
// across a warp and every thread has the same share of R copies.
constexpr int kIntraThreads = 256;
// Waits of the intra kernel (inputs, products) let the waiting warps sleep up to
// this long per try, so that they leave the issue slots to the SM's other CTA.
constexpr uint32_t kIntraSuspendNs = 20000;
constexpr uint32_t kRawTile = kChunk * kDK * 2;    // one [64][128] bf16 tile, 16 KiB
// Shared memory (offsets from a 1024-aligned base).  The raw k, q, v, z tiles
// arrive by two 128-byte-swizzled TMA boxes each (one per K half of 64
// channels), as K-major operand images of 64 rows x 128 B.  k and q are
// interleaved by K half, [k K0 | q K0 | k K1 | q K1], so that after pass 2 each
// K half holds the 128-row operand [K e^L; Q e^L] of the A/P product:
// element (r, c) of k at kq_offset(r, c), of q 8 KiB further.  v and z are
// [K0 | K1]: element (r, c) at sw128_offset(r, c, 64).
constexpr uint32_t kRawK = 0, kRawQ = 8192, kRawV = 2 * kRawTile, kRawZ = 3 * kRawTile;
__host__ __device__ __forceinline__ uint32_t kq_offset(uint32_t r, uint32_t c) {
    return (c >> 6) * 16384u + sw128_offset(r, c & 63, 64);
}
// B operand of the A/P product: the images R^(I) = k e^{m_I - G} (rows 0 ..
// 16 I + 15, scaled to sub-tile I's reference) stacked per K half, 16 + 32 + 48
// + 64 = 160 rows of 128 B: R^(I) starts at row 8 I (I + 1).
constexpr uint32_t kIR = 4 * kRawTile;
constexpr uint32_t kRStack = 160 * 128;             // one K half of the stack: 20 KiB
__host__ __device__ constexpr uint32_t r_region(int I, int kb) {
    return kIR + (uint32_t)kb * kRStack + 1024u * (uint32_t)(I * (I + 1));
}
constexpr uint32_t kISmem = kIR + 40960;           // 104 KiB
// Reused inside the R area once the A/P products are read back:
// (rows padded to 68 and 36 floats: 16-byte aligned for vector loads)
constexpr int kLd = 68, kXLd = 36;
constexpr uint32_t kIAf = kIR;                     // fp32 A [64][68]
constexpr uint32_t kITf = kIR + 64 * kLd * 4;      // fp32 T [64][68]
constexpr uint32_t kIXf = kIR + 128 * kLd * 4;     // fp32 scratch [32][36]
static_assert(kIXf + 32 * kXLd * 4 <= kIR + 40960, "inverse scratch exceeds the R area");
// Later uses of the raw tiles within an item:
//   k and q: K e^{L}, Q e^{L} (in place), the A operand of the A/P product; then
//           its first 8 KiB hold T as bf16 operand of the W/U product, the next
//           8 KiB the P staging for its bulk store;
//   v, z tiles: [beta K e^G ; beta V]^T, the B operand of the W/U product.
// Once the W/U product completes no tile is read any more, so the next item's
// loads are issued then and overlap the W/U readback (which writes W and U to
// the block straight from registers).

struct IntraItem { int t0, len, g, h; };

// One 3-D tile load: the box {64 channels, 1 head, 64 tokens} at (x, h, t0) of a
// [T][H][128] bf16 tensor, 128-byte swizzled; rows past T arrive as zeros.
__device__ __forceinline__ void tma_rows(void *smem_dst, const CUtensorMap *map, int x, int h,
                                         int t0, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];"
        ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(h), "r"(t0),
          "r"(smem_u32(bar))
        : "memory");
}

// Prefetch of the same box into L2 (no shared memory, no completion).
__device__ __forceinline__ void tma_prefetch_rows(const CUtensorMap *map, int x, int h, int t0) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(h), "r"(t0)
                 : "memory");
}

__device__ __forceinline__ void compute_sync() { __syncthreads(); }

__device__ __forceinline__ void cp_async_4(void *smem_dst, const void *gmem_src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_8(void *smem_dst, const void *gmem_src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ float2 ld_bf16x2_smem(const uint8_t *base, uint32_t off) {
    return __bfloat1622float2(*(const __nv_bfloat162 *)(base + off));
}


// The gate with the fast exponential and division (a few ulp; the bf16 path's
// tolerance is far looser).  Limits as in gate_log_decay: exp(A) z -> +inf gives
// g_min, -> -inf gives 0 (1 / +inf through the fast division is 0).
// Packed fp32 pair arithmetic (one f32x2 instruction for both lanes of a
// channel pair; each lane is an IEEE round-to-nearest operation) and the
// approximate base-2 exponential and reciprocal of the special-function unit.
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 sub2(float2 a, float2 b) { return __fadd2_rn(a, make_float2(-b.x, -b.y)); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float2 exp2_2(float2 x) { return make_float2(ex2_approx(x.x), ex2_approx(x.y)); }
constexpr float kLog2e = 1.4426950408889634f;
__device__ __forceinline__ float2 log2e2() { return make_float2(kLog2e, kLog2e); }
__device__ __forceinline__ uint32_t pack2(float2 v) { return pack_bf16(v.x, v.y); }

// The gate with the approximate exponential and reciprocal (a few ulp; the
// bf16 path's tolerance is far looser), given eAn = -exp(A) log2(e):
// g = g_min / (1 + 2^{eAn z}).  Limits as in gate_log_decay: exp(A) z -> +inf
// gives 2^{-inf} = 0 and g = g_min; -> -inf gives 1 / inf = 0, i.e. g = -0.
__device__ __forceinline__ float gate_fast(float eAn, float z) {
    return kGMin * rcp_approx(1.0f + ex2_approx(eAn * z));
}
__device__ __forceinline__ float2 gate2(float2 eAn, float2 z) {
    const float2 d = add2(exp2_2(mul2(eAn, z)), make_float2(1.f, 1.f));
    return mul2(make_float2(rcp_approx(d.x), rcp_approx(d.y)), make_float2(kGMin, kGMin));
}

__device__ __forceinline__ float lg2_approx(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
constexpr float kLn2 = 0.6931471805599453f;

// The unbounded gate g = -softplus(exp(A) z) = -(max(x, 0) + ln(1 + e^{-|x|})),
// x = exp(A) z, with the approximate exponential and logarithm (absolute error
// of a few 1e-7), clamped at kGClampSoftplus like the exact form.
__device__ __forceinline__ float gate_softplus_fast(float eA, float z) {
    const float x = eA * z;
    const float l1p = kLn2 * lg2_approx(1.0f + ex2_approx(-fabsf(x) * kLog2e));
    return fmaxf(-(fmaxf(x, 0.0f) + l1p), kGClampSoftplus);
}

// GATE = kGateBounded: the K3 gate, dense diagonal tiles (the bound keeps every
// factor below e^80).  GATE = kGateSoftplus: the unbounded gate; the diagonal
// 16 x 16 tiles of A and P come from diag_pair_kernel (`pairs`), their R rows
// are zero, and every other factor is formed as one exponent <= 0.
template <int GATE>
__global__ void __launch_bounds__(kIntraThreads, 2)
intra_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_z,
             const float *__restrict__ A, const float *__restrict__ beta,
             const int2 *__restrict__ chunk_loc, const int32_t *__restrict__ chunk_off, int N, int H,
             uint8_t *__restrict__ blocks, int64_t max_chunks, int32_t *status,
             const float *__restrict__ pairs)
{
    constexpr bool kSoftplus = GATE == kGateSoftplus;
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = align_smem_1024(smraw);
    __shared__ uint64_t full, mma_bar, ap_bar;
    __shared__ uint32_t tbase;
    __shared__ IntraItem info;
    __shared__ int2 next_loc;
    __shared__ float sBeta[kChunk];
    __shared__ float sA[kDK];
    __shared__ float sHalf[8][kDK];   // gate sums of the eight 8-row half-blocks
    __shared__ volatile int sAbort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int total_items = chunk_off[N] * H;
    if ((int)blockIdx.x >= total_items) return;
    if (tid == 0) {
        mbar_init(&full, 1);
        mbar_init(&mma_bar, 1);
        mbar_init(&ap_bar, 1);
        fence_mbar_init();
        sAbort = 0;
    }
    if (warp == 0) { tmem_alloc(&tbase, 256); tmem_relinquish(); }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tb = tbase;

    // Where item wn lives (one load of the plan's chunk table).
    auto locate = [&](int wn) {
        const int g = wn / H, h = wn % H;
        const int2 loc = chunk_loc[g];
        return IntraItem{loc.x, loc.y, g, h};
    };
    // Warp 0: request item `nx` (raw rows by eight TMA boxes, beta and A by
    // cp.async).  Called once the previous item reads no raw tile, beta or A.
    auto issue = [&](const IntraItem &nx) {
        for (int r = lane; r < kChunk; r += 32) {
            if (r < nx.len) cp_async_4(&sBeta[r], beta + (size_t)(nx.t0 + r) * H + nx.h);
            else sBeta[r] = 0.f;
        }
        for (int c = lane; c < kDK; c += 32) cp_async_4(&sA[c], A + (size_t)nx.h * kDK + c);
        cp_async_commit();
        if (lane == 0) {
            info = nx;
            mbar_arrive_expect_tx(&full, 4 * kRawTile);
            const CUtensorMap *maps[4] = {&tm_k, &tm_q, &tm_v, &tm_z};
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                // k, q: K halves 16 KiB apart (interleaved); v, z: 8 KiB apart.
                const uint32_t base = m < 2 ? 8192u * m : kRawTile * m;
                const uint32_t kh1 = m < 2 ? 16384u : 8192u;
                tma_rows(sm + base, maps[m], 0, nx.h, nx.t0, &full);
                tma_rows(sm + base + kh1, maps[m], 64, nx.h, nx.t0, &full);
            }
        }
        __syncwarp();
    };
    if (warp == 0) issue(locate(blockIdx.x));
    int issued = 1;  // items requested so far (meaningful in warp 0)

    {
        const int cp = ((warp & 1) << 5) | lane, c0 = 2 * cp, p = warp >> 1;
        float *Af = (float *)(sm + kIAf), *Tf = (float *)(sm + kITf), *Xf = (float *)(sm + kIXf);
        uint32_t mma_count = 0;
        int mma_failed = -1, ap_failed = -1;  // parity of a product wait that gave up
        int it = 0;
        for (int w = blockIdx.x; w < total_items && !sAbort; w += gridDim.x, ++it) {
            // Warp 0 alone waits for the item's inputs (its own cp.async of beta and A,
            // and the TMA boxes); the other warps wait at the barrier, where they take
            // no issue slots from the SM's other CTA.
            if (warp == 0) {
                cp_async_wait_all();
                if (!mbar_wait<kIntraSuspendNs>(&full, it & 1, globaltimer_ns() + kWaitNs)) {
                    if (lane == 0) record_timeout(status);
                    sAbort = 1;
                }
            }
            compute_sync();  // inputs landed, beta and A visible to every warp
            tc_fence_after_sync();  // the previous item's TMEM reads precede this item's writes
            const IntraItem inf = info;
            const int len = inf.len, h = inf.h;
            uint8_t *blk = blocks + ((size_t)h * max_chunks + inf.g) * kBlockBytes;
            // exp(A) of channels c0, c0 + 1; for the bounded gate pre-multiplied by
            // -log2(e), the form gate2 takes.
            const float2 eA2 = exp2_2(mul2(*(const float2 *)&sA[c0], log2e2()));
            const float2 eAn = kSoftplus ? eA2 : mul2(eA2, make_float2(-kLog2e, -kLog2e));
            const bool has_next = w + (int)gridDim.x < total_items;
            // The next item's chunk-table entry, fetched asynchronously for issue().
            if (tid == 0 && has_next) {
                cp_async_8(&next_loc, chunk_loc + (w + gridDim.x) / H);
                cp_async_commit();
            }

            // Pass 1: gate of channels c0, c0 + 1 over two 8-row half-blocks, b = p and
            // b = 7 - p (p = warp / 2).  Half-block b lies in sub-tile b / 2, whose rows
            // are copied into 4 - b / 2 of the R images in pass 2, so this pairing gives
            // every thread the same number of copies.  Each row's running sum from its
            // half-block start is parked in TMEM for pass 2 (lane 32 (warp % 4) + lane,
            // 16 columns per half-block from 128 + 32 (warp / 4)); those columns are free
            // from the previous item's W/U readback until this item's W/U product.
            // beta V of the same rows is formed here too, so that the v tile is dead
            // after this pass.
            const uint32_t lcol = tmem_addr(tb, 32 * (warp & 3), 128 + 32 * (warp >> 2));
            uint32_t pv0[8], pv1[8];   // beta V, rows (2 m, 2 m + 1) of channel c0 / c0 + 1
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int b = q == 0 ? p : 7 - p;
                float2 acc = make_float2(0.f, 0.f);
                float lst[8];
                float2 hv[2];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = 8 * b + i;
                    const uint32_t so = sw128_offset(r, c0, 64);
                    float2 vv = make_float2(0.f, 0.f);
                    if (r < len) {
                        const float2 zz = ld_bf16x2_smem(sm, kRawZ + so);
                        acc = add2(acc, kSoftplus ? make_float2(gate_softplus_fast(eAn.x, zz.x),
                                                                gate_softplus_fast(eAn.y, zz.y))
                                                  : gate2(eAn, zz));
                        vv = ld_bf16x2_smem(sm, kRawV + so);
                    }
                    hv[i & 1] = mul2(vv, make_float2(sBeta[r], sBeta[r]));
                    if (i & 1) {
                        pv0[4 * q + (i >> 1)] = pack_bf16(hv[0].x, hv[1].x);
                        pv1[4 * q + (i >> 1)] = pack_bf16(hv[0].y, hv[1].y);
                    }
                    lst[2 * (i & 3)] = acc.x;
                    lst[2 * (i & 3) + 1] = acc.y;
                    if ((i & 3) == 3) tmem_st8(lcol + 16 * q + 8 * (i >> 2), lst);
                }
                *(float2 *)&sHalf[b][c0] = acc;
            }
            tmem_st_wait();
            compute_sync();
            if (sAbort) break;
            if (tid == 0 && has_next) {
                // The next item's rows into L2 now, so that its tile loads (issued once
                // this item's W/U product is done) come from L2.
                cp_async_wait_all();
                const int2 loc = next_loc;
                const int hn = (w + (int)gridDim.x) % H;
                const CUtensorMap *maps[4] = {&tm_k, &tm_q, &tm_v, &tm_z};
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    tma_prefetch_rows(maps[m], 0, hn, loc.x);
                    tma_prefetch_rows(maps[m], 64, hn, loc.x);
                }
            }
            // (beta V)^T (rows = channels, K = tokens) into the z tile, dead since pass
            // 1: rows 128..255 of the B operand of the W/U product.
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int kk = 8 * (q == 0 ? p : 7 - p);
                *(uint4 *)(sm + kRawZ + sw128_offset(c0, kk, 128)) =
                    make_uint4(pv0[4 * q], pv0[4 * q + 1], pv0[4 * q + 2], pv0[4 * q + 3]);
                *(uint4 *)(sm + kRawZ + sw128_offset(c0 + 1, kk, 128)) =
                    make_uint4(pv1[4 * q], pv1[4 * q + 1], pv1[4 * q + 2], pv1[4 * q + 3]);
            }
            // G_C = the sum of the eight half-blocks; e^{G_C} goes to the block
            // (warps 0 and 1 hold channels 0..127 between them).
            float2 GC = make_float2(0.f, 0.f);
#pragma unroll
            for (int b = 0; b < 8; ++b) GC = add2(GC, *(const float2 *)&sHalf[b][c0]);
            if (warp < 2) *(float2 *)(blk + kOffDecay + 4 * c0) = exp2_2(mul2(GC, log2e2()));

            // Pass 2, per half-block: scaled operands of channels c0, c0 + 1 for its 8
            // rows, with L = G - m_I read back from TMEM four rows at a time.
            // Kt = k e^{L} and Qt = q e^{L} replace k and q in place (same thread, same
            // address); the R copies, Q e^{G} and K e^{G_C - G} (to the block) and
            // (beta K e^{G})^T (into the v tile, dead since pass 1) are written as soon
            // as they are formed.
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int b = q == 0 ? p : 7 - p, I = b >> 1;
                // Sub-tile references m_J = G at the end of sub-tile J - 1 (m_0 = 0):
                // m_I, and fac[Ip] = e^{m_Ip - m_I} for the later sub-tiles Ip > I, which
                // carries a column operand from sub-tile I's reference to Ip's.
                float2 mI = make_float2(0.f, 0.f), fac[4];
                {
                    float2 m = make_float2(0.f, 0.f);
#pragma unroll
                    for (int J = 0; J < 4; ++J) {
                        if (J == I) mI = m;
                        fac[J] = m;
                        m = add2(m, add2(*(const float2 *)&sHalf[2 * J][c0], *(const float2 *)&sHalf[2 * J + 1][c0]));
                    }
                }
                // Bounded gate: fac[J] = e^{m_J - m_I}.  Unbounded gate: fac[J] = m_J - m_I
                // (<= 0), added to -L inside one exponent per copy instead.
#pragma unroll
                for (int J = 1; J < 4; ++J)
                    fac[J] = kSoftplus ? sub2(fac[J], mI) : exp2_2(mul2(sub2(fac[J], mI), log2e2()));
                const float2 off = (b & 1) ? *(const float2 *)&sHalf[b - 1][c0] : make_float2(0.f, 0.f);
                const float2 emI = exp2_2(mul2(mI, log2e2()));
                const float2 gcm = sub2(GC, mI);
                const float2 egc = kSoftplus ? gcm : exp2_2(mul2(gcm, log2e2()));
                uint32_t pk0[4], pk1[4], kd0[4], kd1[4];
                float lrd[16];  // partial sums of the half-block's 8 rows, from pass 1
                tmem_ld16f(lcol + 16 * q, lrd);
                tmem_ld_wait();
#pragma unroll
                for (int i2 = 0; i2 < 8; i2 += 2) {
                    float2 hk[2], hd[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int i = i2 + u, r = 8 * b + i;
                        const bool valid = r < len;
                        const uint32_t so = kq_offset(r, c0);
                        const float2 L = add2(make_float2(lrd[2 * i], lrd[2 * i + 1]), off);
                        const float2 kv = valid ? ld_bf16x2_smem(sm, kRawK + so) : make_float2(0.f, 0.f);
                        const float2 qv = valid ? ld_bf16x2_smem(sm, kRawQ + so) : make_float2(0.f, 0.f);
                        const float2 lg = mul2(L, log2e2());
                        const float2 e1 = exp2_2(lg);                          // in [e^-80, 1]
                        const float br = sBeta[r];
                        const float2 kt = mul2(kv, e1), qt = mul2(qv, e1);
                        *(uint32_t *)(sm + kRawK + so) = pack2(kt);
                        *(uint32_t *)(sm + kRawQ + so) = pack2(qt);
                        const uint32_t ro = sw128_offset(r, c0 & 63, 64);
                        if constexpr (kSoftplus) {
                            // Diagonal tile rows are zero (the pair kernel supplies that
                            // tile); later sub-tiles get k e^{m_Ip - G} as one exponent.
                            *(uint32_t *)(sm + r_region(I, c0 >> 6) + ro) = 0u;
#pragma unroll
                            for (int Ip = 1; Ip < 4; ++Ip)
                                if (Ip > I)
                                    *(uint32_t *)(sm + r_region(Ip, c0 >> 6) + ro) =
                                        pack2(mul2(kv, exp2_2(mul2(sub2(fac[Ip], L), log2e2()))));
                            hd[u] = mul2(kv, exp2_2(mul2(sub2(egc, L), log2e2())));
                        } else {
                            const float2 kb = mul2(kv, exp2_2(make_float2(-lg.x, -lg.y)));  // [1, e^80]
                            *(uint32_t *)(sm + r_region(I, c0 >> 6) + ro) = pack2(kb);
#pragma unroll
                            for (int Ip = 1; Ip < 4; ++Ip)
                                if (Ip > I)
                                    *(uint32_t *)(sm + r_region(Ip, c0 >> 6) + ro) = pack2(mul2(kb, fac[Ip]));
                            hd[u] = mul2(kb, egc);
                        }
                        *(uint32_t *)(blk + kOffWQ + sw128_offset(64 + r, c0, 128)) = pack2(mul2(qt, emI));
                        hk[u] = mul2(mul2(kt, emI), make_float2(br, br));
                    }
                    // Rows i2, i2 + 1 of each channel as one bf16 pair (low half = row i2).
                    pk0[i2 >> 1] = pack_bf16(hk[0].x, hk[1].x);
                    pk1[i2 >> 1] = pack_bf16(hk[0].y, hk[1].y);
                    kd0[i2 >> 1] = pack_bf16(hd[0].x, hd[1].x);
                    kd1[i2 >> 1] = pack_bf16(hd[0].y, hd[1].y);
                }
                // (beta K e^G)^T into the v tile: rows 0..127 of the W/U product's B
                // operand; (K e^{G_C - G})^T straight to its block region (rows =
                // channels, K = tokens 8 b .. 8 b + 7, the state kernel's B operand).
                const int kk = 8 * b;
                *(uint4 *)(sm + kRawV + sw128_offset(c0, kk, 128)) = make_uint4(pk0[0], pk0[1], pk0[2], pk0[3]);
                *(uint4 *)(sm + kRawV + sw128_offset(c0 + 1, kk, 128)) = make_uint4(pk1[0], pk1[1], pk1[2], pk1[3]);
                *(uint4 *)(blk + kOffKd + kd_offset(c0, kk)) = make_uint4(kd0[0], kd0[1], kd0[2], kd0[3]);
                *(uint4 *)(blk + kOffKd + kd_offset(c0 + 1, kk)) = make_uint4(kd1[0], kd1[1], kd1[2], kd1[3]);
            }

            // A/P product, one M = 128, N = 160 product over both K halves:
            //   D[r][8 I (I + 1) + s]      = Kt_r . R^(I)_s   (r < 64: A before beta)
            //   D[64 + r][8 I (I + 1) + s] = Qt_r . R^(I)_s   (P),
            // of which the readback takes, for row r of sub-tile I, its own image's
            // columns.  Eight tensor-core instructions for all four sub-tiles.
            fence_proxy_async_smem();
            tc_fence_before_sync();
            compute_sync();
            tc_fence_after_sync();
            if (warp == 0) {
                if (elect_one()) {
                    const uint32_t id = idesc_bf16_f32(128, 160), base = smem_u32(sm);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_ss(tmem_addr(tb, 0, 0),
                               desc_kmajor_sw128(base + (ks >> 2) * 16384 + (ks & 3) * 32),
                               desc_kmajor_sw128(base + kIR + (ks >> 2) * kRStack + (ks & 3) * 32), id,
                               ks > 0);
                    mma_commit(&ap_bar);
                }
                __syncwarp();
            }
            if (warp == 0 && !mbar_wait<kIntraSuspendNs>(&ap_bar, it & 1, globaltimer_ns() + kWaitNs)) {
                if (lane == 0) record_timeout(status);
                sAbort = 1;
                ap_failed = it & 1;
            }
            compute_sync();  // the A/P products are complete (observed by warp 0)
            tc_fence_after_sync();
            {
                // Warp w: lane quarter qd = w % 4 holds rows r = 32 (qd % 2) + lane of A
                // (qd < 2) or of P (qd >= 2); half hw = w / 4 takes columns s = 32 hw ..
                // 32 hw + 31 of those rows, in two groups of 16 whose four loads share
                // one wait.  The two half-warps' rows lie in different sub-tiles, whose
                // images start at different D columns, so each group is loaded at both
                // bases and every lane keeps its own.
                const int qd = warp & 3, hw = warp >> 2;
                const int r = 32 * (qd & 1) + lane, Ia = r >> 4;
                const int I0 = 2 * (qd & 1);
                const uint32_t nlo = 8u * I0 * (I0 + 1), nhi = 8u * (I0 + 1) * (I0 + 2);
                const uint32_t lrow = tmem_addr(tb, 32 * qd, 0);
                const bool isP = qd >= 2;
                const float br = sBeta[r];
                float va2[2][16], vb2[2][16];
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    tmem_ld16f(lrow + nlo + 32 * hw + 16 * g, va2[g]);
                    tmem_ld16f(lrow + nhi + 32 * hw + 16 * g, vb2[g]);
                }
                tmem_ld_wait();
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    const int s0 = 32 * hw + 16 * g;
                    float v[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[e] = lane < 16 ? va2[g][e] : vb2[g][e];
                    if (kSoftplus && 2 * hw + g == Ia) {
                        // The diagonal tile, from the pair kernel: [A | P][I][r][s] per item.
                        const float4 *pa = (const float4 *)(pairs + ((size_t)h * max_chunks + inf.g) * 2048 +
                                                            (isP ? 1024 : 0) + Ia * 256 + (r & 15) * 16);
#pragma unroll
                        for (int v4 = 0; v4 < 4; ++v4) {
                            const float4 x = pa[v4];
                            v[4 * v4] = x.x; v[4 * v4 + 1] = x.y; v[4 * v4 + 2] = x.z; v[4 * v4 + 3] = x.w;
                        }
                    }
                    if (!isP) {
                        // A = strictly_lower(Diag(beta) Kt Kh^T), fp32 rows for the inverse.
#pragma unroll
                        for (int e = 0; e < 16; e += 4)
                            *(float4 *)&Af[r * kLd + s0 + e] =
                                make_float4(s0 + e < r ? br * v[e] : 0.f, s0 + e + 1 < r ? br * v[e + 1] : 0.f,
                                            s0 + e + 2 < r ? br * v[e + 2] : 0.f,
                                            s0 + e + 3 < r ? br * v[e + 3] : 0.f);
                    } else {
                        // P = lower(Qt Kh^T), bf16 operand image rows (the staging of its store).
#pragma unroll
                        for (int e = 0; e < 16; e += 8) {
                            uint32_t w4[4];
#pragma unroll
                            for (int k2 = 0; k2 < 4; ++k2) {
                                const int sa = s0 + e + 2 * k2;
                                w4[k2] = pack_bf16(sa <= r ? v[e + 2 * k2] : 0.f, sa + 1 <= r ? v[e + 2 * k2 + 1] : 0.f);
                            }
                            *(uint4 *)(sm + kRawK + 8192 + sw128_offset(r, s0 + e, 64)) =
                                make_uint4(w4[0], w4[1], w4[2], w4[3]);
                        }
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            compute_sync();
            if (sAbort) break;
            if (tid == 0) {
                bulk_s2g(blk + kOffP, sm + kRawK + 8192, 8192);
                bulk_commit();
            }

            // T = (I + A)^-1 by blocks of 16: diagonal blocks by forward
            // substitution, then T_ij = -T_ii A_ij T_jj doubled from 16 to 32 to 64.
            // Only the lower triangle is used; the two upper blocks that the
            // doubling products read, (0,1) and (2,3), are set to zero.  T, rounded
            // to bf16, is also the A operand of the W/U product (64 rows x 64 K),
            // written into the k tile as it is formed.
            uint8_t *sT = sm + kRawK;
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
                // The other 192 threads zero the upper blocks, one 16-byte store each:
                // (0,1) (0,2) (0,3) (1,2) (1,3) (2,3) of the bf16 operand, 16 rows x 2
                // chunks of 8 each, and (0,1), (2,3) of the fp32 T that the doubling
                // products read, 16 rows x 4 float4 each.
                const int e = tid - 64;
                {
                    const int bz = e >> 5, r = (e >> 1) & 15, hf = e & 1;
                    const int bi = bz < 3 ? 0 : bz < 5 ? 1 : 2;
                    const int bj = bz < 3 ? bz + 1 : bz < 5 ? bz - 1 : 3;
                    *(uint4 *)(sT + sw128_offset(16 * bi + r, 16 * bj + 8 * hf, 64)) = make_uint4(0u, 0u, 0u, 0u);
                }
                if (e < 128) {
                    const int blkz = e >> 6, r = (e >> 2) & 15, c4 = e & 3;
                    *(float4 *)&Tf[(32 * blkz + r) * kLd + 32 * blkz + 16 + 4 * c4] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
            compute_sync();
            {
                // Level 1, blocks (1,0) and (3,2): X = A_ij T_jj, then T_ij = -T_ii X.
                // Warps 0-3: thread (pb, r, cb) computes rows r and r + 8 x columns
                // cb, cb + 1 of block pair pb (one float2 of the right factor per two rows).
                const int pb = (tid >> 6) & 1, r = (tid >> 3) & 7, cb = 2 * (tid & 7);
                const int oi = 32 * pb + 16, oj = 32 * pb;
                const bool act = tid < 128;
                if (act) {
                    float2 x0 = make_float2(0.f, 0.f), x1 = x0;
#pragma unroll
                    for (int t = 0; t < 16; ++t) {
                        const float a = Af[(oi + r) * kLd + oj + t], a2 = Af[(oi + r + 8) * kLd + oj + t];
                        const float2 tv = *(const float2 *)&Tf[(oj + t) * kLd + oj + cb];
                        x0 = fma2(make_float2(a, a), tv, x0);
                        x1 = fma2(make_float2(a2, a2), tv, x1);
                    }
                    *(float2 *)&Xf[(16 * pb + r) * kXLd + cb] = x0;
                    *(float2 *)&Xf[(16 * pb + r + 8) * kXLd + cb] = x1;
                }
                compute_sync();
                if (act) {
                    float2 y0 = make_float2(0.f, 0.f), y1 = y0;
#pragma unroll
                    for (int t = 0; t < 16; ++t) {
                        const float tt = Tf[(oi + r) * kLd + oi + t], tt2 = Tf[(oi + r + 8) * kLd + oi + t];
                        const float2 xv = *(const float2 *)&Xf[(16 * pb + t) * kXLd + cb];
                        y0 = fma2(make_float2(tt, tt), xv, y0);
                        y1 = fma2(make_float2(tt2, tt2), xv, y1);
                    }
                    *(float2 *)&Tf[(oi + r) * kLd + oj + cb] = make_float2(-y0.x, -y0.y);
                    *(float2 *)&Tf[(oi + r + 8) * kLd + oj + cb] = make_float2(-y1.x, -y1.y);
                    *(uint32_t *)(sT + sw128_offset(oi + r, oj + cb, 64)) = pack_bf16(-y0.x, -y0.y);
                    *(uint32_t *)(sT + sw128_offset(oi + r + 8, oj + cb, 64)) = pack_bf16(-y1.x, -y1.y);
                }
            }
            compute_sync();
            {
                // Level 2, block rows 32..63 x columns 0..31.  Warps 0-3: each thread
                // computes rows r and r + 16 x columns cb .. cb + 3 of each product, so
                // that one float4 of the right factor serves two rows (the products are
                // bound by shared-memory reads).
                const int r = (tid >> 3) & 15, cb = 4 * (tid & 7);
                const bool act = tid < 128;
                if (act) {
                    float2 x0 = make_float2(0.f, 0.f), x1 = x0, x2 = x0, x3 = x0;
#pragma unroll
                    for (int t = 0; t < 32; ++t) {
                        const float a = Af[(32 + r) * kLd + t], a2 = Af[(48 + r) * kLd + t];
                        const float4 tv = *(const float4 *)&Tf[t * kLd + cb];
                        const float2 lo = make_float2(tv.x, tv.y), hi = make_float2(tv.z, tv.w);
                        x0 = fma2(make_float2(a, a), lo, x0);
                        x1 = fma2(make_float2(a, a), hi, x1);
                        x2 = fma2(make_float2(a2, a2), lo, x2);
                        x3 = fma2(make_float2(a2, a2), hi, x3);
                    }
                    *(float4 *)&Xf[r * kXLd + cb] = make_float4(x0.x, x0.y, x1.x, x1.y);
                    *(float4 *)&Xf[(r + 16) * kXLd + cb] = make_float4(x2.x, x2.y, x3.x, x3.y);
                }
                compute_sync();
                if (act) {
                    float2 y0 = make_float2(0.f, 0.f), y1 = y0, y2 = y0, y3 = y0;
#pragma unroll
                    for (int t = 0; t < 32; ++t) {
                        const float tt = Tf[(32 + r) * kLd + 32 + t], tt2 = Tf[(48 + r) * kLd + 32 + t];
                        const float4 xv = *(const float4 *)&Xf[t * kXLd + cb];
                        const float2 lo = make_float2(xv.x, xv.y), hi = make_float2(xv.z, xv.w);
                        y0 = fma2(make_float2(tt, tt), lo, y0);
                        y1 = fma2(make_float2(tt, tt), hi, y1);
                        y2 = fma2(make_float2(tt2, tt2), lo, y2);
                        y3 = fma2(make_float2(tt2, tt2), hi, y3);
                    }
                    *(uint2 *)(sT + sw128_offset(32 + r, cb, 64)) =
                        make_uint2(pack_bf16(-y0.x, -y0.y), pack_bf16(-y1.x, -y1.y));
                    *(uint2 *)(sT + sw128_offset(48 + r, cb, 64)) =
                        make_uint2(pack_bf16(-y2.x, -y2.y), pack_bf16(-y3.x, -y3.y));
                }
            }
            // The Kd^T and P staging is read out before the next item's loads land on it.
            if (tid == 0) bulk_wait_read<0>();
            fence_proxy_async_smem();
            tc_fence_before_sync();
            compute_sync();
            tc_fence_after_sync();
            if (tid == 0) {
                // [W | U] = T [beta K e^G | beta V]  (M = 64, N = 256, K = 64)
                const uint32_t id = idesc_bf16_f32(64, 256);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_ss(tmem_addr(tb, 0, 0), desc_kmajor_sw128(smem_u32(sT) + ks * 32),
                           desc_kmajor_sw128(smem_u32(sm + kRawV) + ks * 32), id, ks > 0);
                mma_commit(&mma_bar);
            }
            if (warp == 0 && !mbar_wait<kIntraSuspendNs>(&mma_bar, mma_count & 1, globaltimer_ns() + kWaitNs)) {
                if (lane == 0) record_timeout(status);
                sAbort = 1;
                mma_failed = (int)(mma_count & 1);
            }
            ++mma_count;
            compute_sync();  // the W/U product is complete (observed by warp 0)
            tc_fence_after_sync();
            // No raw tile is read any more: the next item's loads overlap the readback.
            if (warp == 0 && has_next && !sAbort) {
                cp_async_wait_all();
                __syncwarp();
                const int wn = w + gridDim.x;
                const int2 loc = next_loc;
                issue(IntraItem{loc.x, loc.y, wn / H, wn % H});
                issued = it + 2;
            }
            {
                // Rows r = 16 q + i (i < 16) of lane quarter q = w % 4; warps 0-3 read W
                // (columns 0..127) into rows 0..63 of the block's [W; Qt] image, warps
                // 4-7 read U (columns 128..255) into its block region.  Each load gives
                // the two threads of a row 16 consecutive columns, so every store
                // instruction writes whole 32-byte sectors (16 rows x 32 B); for U those
                // are 512 contiguous bytes (u_offset).
                const int q = warp & 3, hb = warp >> 2, r = 16 * q + (lane & 15);
#pragma unroll
                for (int m2 = 0; m2 < 8; m2 += 2) {
                    uint32_t rr[2][8];
                    tmem_ld16x2_8(tmem_addr(tb, 32 * q, 128 * hb + 16 * m2), rr[0]);
                    tmem_ld16x2_8(tmem_addr(tb, 32 * q, 128 * hb + 16 * m2 + 16), rr[1]);
                    tmem_ld_wait();
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const uint4 w4 = make_uint4(
                            pack_bf16(__uint_as_float(rr[u][0]), __uint_as_float(rr[u][1])),
                            pack_bf16(__uint_as_float(rr[u][2]), __uint_as_float(rr[u][3])),
                            pack_bf16(__uint_as_float(rr[u][4]), __uint_as_float(rr[u][5])),
                            pack_bf16(__uint_as_float(rr[u][6]), __uint_as_float(rr[u][7])));
                        const int col = 16 * (m2 + u) + 8 * (lane >> 4);
                        if (hb == 0)
                            *(uint4 *)(blk + kOffWQ + sw128_offset(r, col, 128)) = w4;
                        else
                            *(uint4 *)(blk + kOffU + u_offset(r, col)) = w4;
                    }
                }
            }
            tc_fence_before_sync();
            compute_sync();  // TMEM is read out before the next item's products
            if (sAbort) break;
        }
        if (tid == 0) bulk_wait<0>();  // every staged block region has reached memory
        // Drain: every requested copy and product has finished before the CTA exits.
        if (warp == 0) {
            cp_async_wait_all();
            if (lane == 0)
                for (int d = it; d < issued; ++d) mbar_wait(&full, d & 1, globaltimer_ns() + kWaitNs);
        }
        if (tid == 0 && mma_failed >= 0) mbar_wait(&mma_bar, (uint32_t)mma_failed, globaltimer_ns() + kWaitNs);
        if (tid == 0 && ap_failed >= 0) mbar_wait(&ap_bar, (uint32_t)ap_failed, globaltimer_ns() + kWaitNs);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, 256);
}

// ------------------------------------------------------------------- pair --

// The unbounded gate's diagonal tiles, pair by pair ("Kimi K3: Architecture,
// Training, and Million-Token Agentic RL", section 3.3: before the bound,
// diagonal tiles needed a position-pair path).  For the 16-token sub-tile I of
// a (chunk, head) item and rows s <= r in it:
//   A[I][r][s] = sum_c k_rc k_sc e^{L_rc - L_sc},   P[I][r][s] = sum_c q_rc k_sc e^{L_rc - L_sc},
// L the cumulative log-decay from the sub-tile start, one exponent per pair and
// channel, so no factor overflows however fast the state decays (beta and the
// causal masks are applied by the intra kernel, which reads these tiles in place
// of its products' diagonal tiles).  One CTA per item; rows beyond the chunk's
// length give zeros.  Output per item: [A | P][I][r][s], 2 x 4 x 16 x 16 fp32
// (only s <= r is written; the intra kernel masks the rest).
constexpr int kPairThreads = 256;
constexpr int kPairLd = 130;   // fp32 row stride of the staged L, k, q rows
constexpr uint32_t kPairSmem = 3u * kChunk * kPairLd * 4u;

__global__ void __launch_bounds__(kPairThreads)
diag_pair_kernel(const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ q,
                 const __nv_bfloat16 *__restrict__ z, const float *__restrict__ A,
                 const int2 *__restrict__ chunk_loc, const int32_t *__restrict__ chunk_off, int N,
                 int H, int64_t max_chunks, float *__restrict__ pairs)
{
    extern __shared__ float psm[];
    float *Ls = psm, *Ks = psm + kChunk * kPairLd, *Qs = psm + 2 * kChunk * kPairLd;
    const int h = blockIdx.x % H, g = blockIdx.x / H;
    if (g >= chunk_off[N]) return;
    const int2 loc = chunk_loc[g];
    const int tid = threadIdx.x;
    {
        // Thread (rg, cp): channels 2 cp, 2 cp + 1 of sub-tile rg's 16 rows.
        const int cp = tid & 63, rg = tid >> 6, c0 = 2 * cp;
        const float eA0 = ex2_approx(A[(size_t)h * kDK + c0] * kLog2e);
        const float eA1 = ex2_approx(A[(size_t)h * kDK + c0 + 1] * kLog2e);
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll 4
        for (int i = 0; i < 16; ++i) {
            const int r = 16 * rg + i;
            float2 kv = make_float2(0.f, 0.f), qv = kv;
            if (r < loc.y) {
                const size_t idx = ((size_t)(loc.x + r) * H + h) * kDK + c0;
                const float2 zz = __bfloat1622float2(*(const __nv_bfloat162 *)(z + idx));
                kv = __bfloat1622float2(*(const __nv_bfloat162 *)(k + idx));
                qv = __bfloat1622float2(*(const __nv_bfloat162 *)(q + idx));
                acc = add2(acc, make_float2(gate_softplus_fast(eA0, zz.x), gate_softplus_fast(eA1, zz.y)));
            }
            *(float2 *)&Ls[r * kPairLd + c0] = acc;
            *(float2 *)&Ks[r * kPairLd + c0] = kv;
            *(float2 *)&Qs[r * kPairLd + c0] = qv;
        }
    }
    __syncthreads();
    float *out = pairs + ((size_t)h * max_chunks + g) * 2048;
    // 4 x 136 (s <= r) pairs; pair index e within a sub-tile: r (r + 1) / 2 + s.
    for (int pidx = tid; pidx < 4 * 136; pidx += kPairThreads) {
        const int I = pidx / 136, e = pidx - 136 * I;
        int r = 0;
        while ((r + 1) * (r + 2) / 2 <= e) ++r;
        const int s = e - r * (r + 1) / 2;
        const float *lr = Ls + (16 * I + r) * kPairLd, *ls = Ls + (16 * I + s) * kPairLd;
        const float *kr = Ks + (16 * I + r) * kPairLd, *ks = Ks + (16 * I + s) * kPairLd;
        const float *qr = Qs + (16 * I + r) * kPairLd;
        float2 a = make_float2(0.f, 0.f), pp = a;
#pragma unroll 8
        for (int c = 0; c < kDK; c += 2) {
            const float2 d = mul2(sub2(*(const float2 *)&lr[c], *(const float2 *)&ls[c]), log2e2());
            const float2 kse = mul2(*(const float2 *)&ks[c], exp2_2(d));    // e^{L_r - L_s} <= 1
            a = fma2(*(const float2 *)&kr[c], kse, a);
            pp = fma2(*(const float2 *)&qr[c], kse, pp);
        }
        out[I * 256 + r * 16 + s] = a.x + a.y;
        out[1024 + I * 256 + r * 16 + s] = pp.x + pp.y;
    }
}

// ------------------------------------------------------------------ state --

// One CTA of 416 threads per (sequence, head) slot, in three roles:
//   chain  (warps 0-7): the per-chunk state recurrence on CUDA cores.  Thread
//          (j, hh) owns TMEM lane j = value channel j and half hh of the delta
//          rows, state columns and the chunk's key channels.
//   output (warps 8-11): reads O^T of each finished chunk from TMEM, rounds it
//          to bf16 in a staging tile and stores whole token rows (one TMA
//          tensor store per full chunk).
//   issue  (warp 12): every tensor-core product and block load, so that no
//          chain thread spends its time issuing; the hand-offs are mbarriers.
// Per chunk c, the products the state recurrence waits for are issued first,
// and those only the outputs need are queued behind them on the tensor pipe,
// where they run while the chain works on CUDA cores:
//   DW     = S_in^T W^T             (critical; commit -> mma1)
//   DO[b]  = S_in^T Qt^T            (outputs; b = c & 1)
//   Dl^T   = U^T - DW               -> bf16 into TMEM                (chain)
//   S^T   += Dl^T Kd                (critical; commit -> mma2s)
//   DO[b] += Dl^T P^T               (outputs; commit -> mma2o[b], empty[stage])
//   S^T    -> bf16 copy SB[(c + 1) & 1] (the next chunk's A operand),
//             then the fp32 master times the next chunk's e^{G_C}    (chain)
//   O^T    = DO[b] -> o                                               (output)
// The bf16 copy of S is double-buffered so that the output product of chunk c
// still reads S_in(c) while the chain writes S_in(c + 1).
constexpr int kStateThreads = 416;
constexpr int kChainThreads = 256, kOutThreads = 128;
constexpr int kIssueWarp = 12;
constexpr uint32_t kStageBytes = 75776;  // block rounded up to 1 KiB
constexpr int kStages = 2;
constexpr uint32_t kOStage = kStages * kStageBytes;  // 2 x [64][128] bf16 output staging
constexpr uint32_t kStateSmem = kStages * kStageBytes + 2 * 16384 + 1024;
// TMEM columns: fp32 S^T, two bf16 copies of S^T, delta^T (bf16), the W
// product, two output accumulators.
constexpr uint32_t kTS = 0, kTSbf = 128, kTDl = 256, kTDW = 288, kTDO = 352;  // SB[b] = 128 + 64 b,
                                                                               // DO[b] = 352 + 64 b
constexpr int kBarOut = 2;  // named barrier id of the output warps
// L2 prefetch distance of the block stream, in chunks (one ahead of the
// two-stage ring).  Measured on the 32K x 96-head workload: 0.86 ms at 2 or 3
// ahead, 0.94 ms at 6 and 1.13 ms at 8; the 96 chains' prefetched blocks crowd
// the L2 at the longer distances.
constexpr int kPrefetchAhead = 3;

struct StateBars {
    uint64_t full[kStages], empty[kStages];
    uint64_t mma1, mma2s, mma2o[2], do_free[2];
    uint64_t sbf_ready, dl_ready, dec_ready, drain;
};

// Barrier over `nthreads` threads of the CTA (named barrier `id`) that also
// returns whether any of them passed `pred` = true, so a group leaves a loop
// together when one of its threads saw a wait give up.
__device__ __forceinline__ bool group_sync_any(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n"
        " barrier.red.or.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void group_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// One TMA tensor store: the [64 tokens][128 channels] bf16 tile at `smem_src`
// to rows t0 .. t0 + 63 of head h of o (rows past T are not written).
__device__ __forceinline__ void tma_store_rows(const CUtensorMap *map, const void *smem_src, int h,
                                               int t0) {
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];"
        ::"l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(h), "r"(t0), "r"(smem_u32(smem_src))
        : "memory");
}

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

// DUMP: the debug variant that also writes delta (dbg_delta); the production
// instantiation has no trace of it.
template <bool DUMP>
__global__ void __launch_bounds__(kStateThreads, 1)
state_kernel(const __grid_constant__ CUtensorMap tm_o,
             const int32_t *__restrict__ cu, const int32_t *__restrict__ chunk_off,
             const int32_t *__restrict__ order, int N, int H,
             const uint8_t *__restrict__ blocks, int64_t max_chunks,
             const float *S0user, float *Sfuser, __nv_bfloat16 *__restrict__ o, int32_t *status,
             int ckpt_every, const int32_t *__restrict__ ckpt_off, float *__restrict__ ckpts,
             int G, float *__restrict__ Sx, float *__restrict__ Mx, uint8_t *__restrict__ Eimg,
             float *__restrict__ dbg_delta)
{
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = align_smem_1024(smraw);
    __shared__ StateBars bars;
    __shared__ uint32_t tbase;

    const int tid = threadIdx.x, warp = tid >> 5;
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
        for (int s = 0; s < kStages; ++s) { mbar_init(&bars.full[s], 1); mbar_init(&bars.empty[s], 1); }
        mbar_init(&bars.mma1, 1);
        mbar_init(&bars.mma2s, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars.mma2o[b], 1);
            mbar_init(&bars.do_free[b], kOutThreads);
        }
        mbar_init(&bars.sbf_ready, kChainThreads);
        mbar_init(&bars.dl_ready, kChainThreads);
        mbar_init(&bars.dec_ready, kChainThreads);
        mbar_init(&bars.drain, 1);
        fence_mbar_init();
    }
    if (warp == 0) { tmem_alloc(&tbase, 512); tmem_relinquish(); }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tb = tbase;
    const uint8_t *blk0 = blocks + ((size_t)h * max_chunks + chunk_off[n] + cbeg) * kBlockBytes;
    const uint32_t lq = 32 * (warp & 3);

    if (warp == kIssueWarp) {
        // ------------------------------------------------------ issue --
        // The whole warp runs the loop (waits are warp-uniform); one elected
        // lane issues each copy, product and commit.
        const bool leader = elect_one();
        const int leader_lane = __ffs(__ballot_sync(0xffffffffu, leader)) - 1;
        int loads = 0;
        auto load = [&](int c) {
            const int s = c % kStages;
            if (leader) {
                mbar_arrive_expect_tx(&bars.full[s], kBlockBytes);
                bulk_g2s(sm + s * kStageBytes, blk0 + (size_t)c * kBlockBytes, kBlockBytes, &bars.full[s]);
                if (c + kPrefetchAhead < nch)
                    bulk_prefetch_l2(blk0 + (size_t)(c + kPrefetchAhead) * kBlockBytes, kBlockBytes);
            }
            ++loads;
            __syncwarp();
        };
        if (leader)
            for (int c = kStages; c < nch && c < kPrefetchAhead; ++c)
                bulk_prefetch_l2(blk0 + (size_t)c * kBlockBytes, kBlockBytes);
        for (int c = 0; c < nch && c < kStages; ++c) load(c);
        // The leader waits; the result is broadcast, so the warp stays converged
        // and leaves the loop as one when a wait gives up.
        auto wait = [&](uint64_t *bar, uint32_t parity) {
            int r = 1;
            if (leader) {
                r = mbar_wait(bar, parity, globaltimer_ns() + kWaitNs) ? 1 : 0;
                if (!r) record_timeout(status);
            }
            return __shfl_sync(0xffffffffu, r, leader_lane) != 0;
        };
        const uint32_t id64 = idesc_bf16_f32(128, 64), id128 = idesc_bf16_f32(128, 128);
        bool ok = true;
        for (int c = 0; c < nch && ok; ++c) {
            const int s = c % kStages, b = c & 1;
            const uint32_t st = smem_u32(sm + s * kStageBytes);
            const uint32_t sb = tmem_addr(tb, 0, kTSbf + 64 * b);
            const uint32_t dO = tmem_addr(tb, 0, kTDO + 64 * b);
            // Descriptors of this stage's operands (warp-uniform, before any issue).
            uint64_t dW[8], dQ[8], dK[4], dP[4];
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                dW[ks] = desc_kmajor_sw128(st + kOffWQ + (ks >> 2) * 16384 + (ks & 3) * 32);
                dQ[ks] = desc_kmajor_sw128(st + kOffWQ + (ks >> 2) * 16384 + 8192 + (ks & 3) * 32);
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                dK[ks] = desc_kmajor_none(st + kOffKd + kd_offset(0, 16 * ks), kKdLbo, kKdSbo);
                dP[ks] = desc_kmajor_sw128(st + kOffP + ks * 32);
            }
            // DW = S_in^T W^T: needs the block and S_in(c) in bf16.
            ok = wait(&bars.full[s], (c / kStages) & 1) && wait(&bars.sbf_ready, c & 1);
            if (!ok) break;
            tc_fence_after_sync();
            if (leader) {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_ts(tmem_addr(tb, 0, kTDW), sb + 8 * ks, dW[ks], id64, ks > 0);
                mma_commit(&bars.mma1);
            }
            __syncwarp();
            // DO[b] = S_in^T Qt^T once output c - 2 has read DO[b].
            ok = c < 2 || wait(&bars.do_free[b], ((c >> 1) - 1) & 1);
            if (!ok) break;
            tc_fence_after_sync();
            if (leader) {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) mma_ts(dO, sb + 8 * ks, dQ[ks], id64, ks > 0);
            }
            __syncwarp();
            // S^T += Dl^T Kd, then DO[b] += Dl^T P^T: need delta(c) and the decayed master.
            ok = wait(&bars.dl_ready, c & 1) && wait(&bars.dec_ready, c & 1);
            if (!ok) break;
            tc_fence_after_sync();
            if (leader) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_ts(tmem_addr(tb, 0, kTS), tmem_addr(tb, 0, kTDl + 8 * ks), dK[ks], id128, true);
                mma_commit(&bars.mma2s);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_ts(dO, tmem_addr(tb, 0, kTDl + 8 * ks), dP[ks], id64, true);
                mma_commit(&bars.mma2o[b]);
                mma_commit(&bars.empty[s]);
            }
            __syncwarp();
            // Stage s is consumed once these products finish: refill it.
            if (c + kStages < nch) {
                ok = wait(&bars.empty[s], (c / kStages) & 1);
                if (!ok) break;
                load(c + kStages);
            }
        }
        if (leader) {
            // Drain: every issued copy has landed and every product has finished
            // before the CTA may exit (bounded waits).
            for (int d = max(0, loads - kStages); d < loads; ++d)
                mbar_wait(&bars.full[d % kStages], (d / kStages) & 1, globaltimer_ns() + kWaitNs);
            mma_commit(&bars.drain);
            mbar_wait(&bars.drain, 0, globaltimer_ns() + kWaitNs);
        }
        __syncwarp();
    } else if (warp < 8) {
        // ------------------------------------------------------- chain --
        const int j = tid & 127, hh = warp >> 2;
        uint32_t ra[32], rb[32];
        // Every lane waits (each reads what the wait guards); the warp decides as
        // one whether to go on, so the warp-collective TMEM accesses stay converged.
        auto wait = [&](uint64_t *bar, uint32_t parity) {
            const bool r = mbar_wait(bar, parity, globaltimer_ns() + kWaitNs);
            if (!r) record_timeout(status);
            return __all_sync(0xffffffffu, r);
        };
        // Initial state: S^T row j = column j of S0 (this half's 64 key channels):
        // fp32 master pre-multiplied by the first chunk's decay, and the bf16 copy
        // SB[0].  The transition X starts from the identity: X^T row j = e_j.
        const bool nonzero0 = S0 || xmode;
        const float *dec0 = (const float *)(sm + kOffDecay);
        bool ok = !nonzero0 || wait(&bars.full[0], 0);
        __syncwarp();
        for (int q2 = 0; q2 < 2; ++q2) {
            const int c0 = 64 * hh + 32 * q2;
            float sv[32];
#pragma unroll
            for (int i = 0; i < 32; ++i)
                sv[i] = S0 ? S0[sbase + (size_t)(c0 + i) * kDV + j] : (xmode && c0 + i == j ? 1.f : 0.f);
#pragma unroll
            for (int i = 0; i < 32; ++i) ra[i] = __float_as_uint(nonzero0 ? sv[i] * dec0[c0 + i] : 0.f);
            tmem_st32(tmem_addr(tb, lq, kTS + c0), ra);
            uint32_t sbb[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) sbb[i] = pack_bf16(sv[2 * i], sv[2 * i + 1]);
            tmem_st16(tmem_addr(tb, lq, kTSbf + c0 / 2), sbb);
        }
        tmem_st_wait();
        tc_fence_before_sync();
        mbar_arrive(&bars.sbf_ready);
        mbar_arrive(&bars.dec_ready);

        for (int c = 0; c < nch && ok; ++c) {
            const int s = c % kStages;
            const uint8_t *st = sm + s * kStageBytes;
            ok = wait(&bars.full[s], (c / kStages) & 1) && wait(&bars.mma1, c & 1);
            if (!ok) break;
            __syncwarp();
            tc_fence_after_sync();
            // Dl^T[j][r] = U[r][j] - DW[j][r] for this half's 32 rows -> bf16 pairs into
            // TMEM (U = 0 on the transition).
            {
                const uint8_t *Uj = st + kOffU + u_offset(0, j);   // U[r][j] at Uj + 32 r
                tmem_ld32(tmem_addr(tb, lq, kTDW + 32 * hh), ra);
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
                        const float d0 = __bfloat162float(*(const __nv_bfloat16 *)(Uj + 32 * r)) -
                                         __uint_as_float(ra[i]);
                        const float d1v = __bfloat162float(*(const __nv_bfloat16 *)(Uj + 32 * (r + 1))) -
                                          __uint_as_float(ra[i + 1]);
                        dl[i >> 1] = pack_bf16(d0, d1v);
                    }
                }
                tmem_st16(tmem_addr(tb, lq, kTDl + 16 * hh), dl);
                if (DUMP) {
                    // Debug dump: delta as the products consume it (bf16), per token.
                    const int t0c = tbeg + c * kChunk, lenc = min(kChunk, tend - t0c);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int r = 32 * hh + i;
                        const uint32_t pr = dl[i >> 1];
                        const float dv = __uint_as_float((i & 1) ? (pr & 0xFFFF0000u) : (pr << 16));
                        if (r < lenc) dbg_delta[((size_t)(t0c + r) * H + h) * kDV + j] = dv;
                    }
                }
                tmem_st_wait();
            }
            tc_fence_before_sync();
            mbar_arrive(&bars.dl_ready);
            ok = wait(&bars.mma2s, c & 1);
            if (!ok) break;
            __syncwarp();
            tc_fence_after_sync();
            const bool last = (c + 1 == nch);
            // S_out, this half's 64 key channels: two loads, one wait.
            tmem_ld32(tmem_addr(tb, lq, kTS + 64 * hh), ra);
            tmem_ld32(tmem_addr(tb, lq, kTS + 64 * hh + 32), rb);
            tmem_ld_wait();
            if (!last) {
                // Critical: the bf16 copy that the next chunk's first product reads.
                uint32_t sa[16], sbv[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    sa[i] = pack_bf16(__uint_as_float(ra[2 * i]), __uint_as_float(ra[2 * i + 1]));
                    sbv[i] = pack_bf16(__uint_as_float(rb[2 * i]), __uint_as_float(rb[2 * i + 1]));
                }
                const uint32_t sbn = kTSbf + 64 * ((c + 1) & 1) + 32 * hh;
                tmem_st16(tmem_addr(tb, lq, sbn), sa);
                tmem_st16(tmem_addr(tb, lq, sbn + 16), sbv);
                tmem_st_wait();
                tc_fence_before_sync();
                mbar_arrive(&bars.sbf_ready);
            }
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
                break;
            }
            // Off the critical path: the fp32 master times the next chunk's decay,
            // before the product that adds to it (dec_ready).
            const int s1 = (c + 1) % kStages;
            ok = wait(&bars.full[s1], ((c + 1) / kStages) & 1);
            if (!ok) break;
            __syncwarp();
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
            mbar_arrive(&bars.dec_ready);
        }
    } else {
        // ------------------------------------------------------ output --
        const int j = tid - kChainThreads;        // TMEM lane = value channel
        const int Ttot = cu[N];                   // rows past it are clipped by the TMA store
        for (int c = 0; c < nch; ++c) {
            const int b = c & 1;
            const int t0 = tbeg + c * kChunk, len = min(kChunk, tend - t0);
            const bool ok = mbar_wait(&bars.mma2o[b], (c >> 1) & 1, globaltimer_ns() + kWaitNs);
            if (!ok) record_timeout(status);
            __syncwarp();
            tc_fence_after_sync();
            uint32_t oa[32], ob[32];
            tmem_ld32(tmem_addr(tb, lq, kTDO + 64 * b), oa);
            tmem_ld32(tmem_addr(tb, lq, kTDO + 64 * b + 32), ob);
            tmem_ld_wait();
            tc_fence_before_sync();
            mbar_arrive(&bars.do_free[b]);
            // Staging buffer c & 1 is free once the stores issued from it (two
            // chunks ago) have read it; waiting for every earlier store is simpler
            // and costs nothing here.
            if (j == 0) bulk_wait_read<0>();
            __syncwarp();
            if (group_sync_any(kBarOut, kOutThreads, !ok)) break;
            uint8_t *ost = sm + kOStage + (c & 1) * 16384;
            if (eimg) {
                // E rows as the K-major, 128-byte-swizzled A operand of the
                // correction product (two 64-wide K halves of 64 rows each).
                const uint32_t kh = (uint32_t)(j >> 6) * 8192u;
#pragma unroll
                for (int r = 0; r < 32; ++r) {
                    *(__nv_bfloat16 *)(ost + kh + sw128_offset(r, j & 63, 64)) =
                        __float2bfloat16_rn(__uint_as_float(oa[r]));
                    *(__nv_bfloat16 *)(ost + kh + sw128_offset(r + 32, j & 63, 64)) =
                        __float2bfloat16_rn(__uint_as_float(ob[r]));
                }
            } else {
                __nv_bfloat16 *ot = (__nv_bfloat16 *)ost;
#pragma unroll
                for (int r = 0; r < 32; ++r) {
                    ot[r * kDV + j] = __float2bfloat16_rn(__uint_as_float(oa[r]));
                    ot[(r + 32) * kDV + j] = __float2bfloat16_rn(__uint_as_float(ob[r]));
                }
            }
            fence_proxy_async_smem();
            group_sync(kBarOut, kOutThreads);
            if (eimg) {
                if (j == 0) { bulk_s2g(eimg + (size_t)c * kEImg, ost, kEImg); bulk_commit(); }
            } else if (len == kChunk || tend == Ttot) {
                if (j == 0) { tma_store_rows(&tm_o, ost, h, t0); bulk_commit(); }
            } else {
                // A ragged last chunk inside the packed batch: plain stores of its rows.
                for (int e = j; e < len * 16; e += kOutThreads) {
                    const int r = e >> 4, part = e & 15;
                    *(uint4 *)(o + ((size_t)(t0 + r) * H + h) * kDV + 8 * part) =
                        *(const uint4 *)(ost + (r * kDV + 8 * part) * 2);
                }
            }
        }
        if (j == 0) bulk_wait<0>();   // every store has completed before the CTA exits
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, 512);
}

// ---------------------------------------------------------------- compose --

// Affine composition of the segments of one (sequence, head), for 16 value
// channels per CTA (columns of S never mix):
//   S_in(1) = S after segment 0,   S_in(s + 1) = M_s S_in(s) + S_loc(s),
// the final state being S_in(Gn).  The whole scan is in fp32; each S_in(s) is
// also written as the bf16 B-operand image (row = value channel, K = key
// channel, 128-byte swizzled) that the correction product reads.  Thread
// (m, half) owns row m and 8 of the CTA's columns.
constexpr int kComposeThreads = 256;
constexpr int kComposeCols = 16;
constexpr int kCpt = kComposeCols / 2;           // columns per thread
constexpr int kMsLd = kDK + 1;
constexpr uint32_t kComposeSmem = (kDK * kMsLd + kDK * kComposeCols) * 4;

__global__ void __launch_bounds__(kComposeThreads)
compose_kernel(const int32_t *__restrict__ chunk_off, int H, int G, const float *__restrict__ Sx,
               const float *__restrict__ Mx, uint8_t *__restrict__ Simg, float *Sf)
{
    extern __shared__ float csm[];
    float *Ms = csm;                 // M_s [128][129]
    float *Ss = csm + kDK * kMsLd;   // S_in(s), this CTA's columns [128][16]
    constexpr int nvb = kDV / kComposeCols;
    const int vb = blockIdx.x % nvb, h = (blockIdx.x / nvb) % H, n = blockIdx.x / (nvb * H);
    const int Gn = min(G, chunk_off[n + 1] - chunk_off[n]);
    if (Gn <= 1) return;             // the state kernel wrote this final state itself
    const int tid = threadIdx.x;
    const int m = tid >> 1, cb = (tid & 1) * kCpt, v0 = vb * kComposeCols;
    auto xoff = [&](int s) { return (((size_t)n * G + s) * H + h) * kStateF32; };

    {   // S_in(1) = state after segment 0: 128 rows x 4 float4 of this CTA's columns
        float4 x[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int e = tid + k * kComposeThreads;
            x[k] = *(const float4 *)(Sx + xoff(0) + (size_t)(e >> 2) * kDV + v0 + 4 * (e & 3));
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) *(float4 *)(Ss + 4 * (tid + k * kComposeThreads)) = x[k];
    }
    __syncthreads();
    for (int s = 1; s < Gn; ++s) {
        // Issue every global load of the step first (one memory latency, not 20).
        float4 mr[16], sl[2];
        const float4 *Mg = (const float4 *)(Mx + xoff(s));
#pragma unroll
        for (int k = 0; k < 16; ++k) mr[k] = Mg[tid + k * kComposeThreads];
        const float4 *Sl = (const float4 *)(Sx + xoff(s) + (size_t)m * kDV + v0 + cb);
#pragma unroll
        for (int k = 0; k < 2; ++k) sl[k] = Sl[k];
        uint8_t *img = Simg + (((size_t)n * G + s) * H + h) * kSinImg;
#pragma unroll
        for (int i = 0; i < kCpt; ++i)
            *(__nv_bfloat16 *)(img + sw128_offset(v0 + cb + i, m, kDV)) =
                __float2bfloat16_rn(Ss[m * kComposeCols + cb + i]);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const int e = tid + k * kComposeThreads;   // float4 index: row e / 32
            float *d = Ms + (e >> 5) * kMsLd + 4 * (e & 31);
            d[0] = mr[k].x; d[1] = mr[k].y; d[2] = mr[k].z; d[3] = mr[k].w;
        }
        __syncthreads();
        float acc[kCpt];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            acc[4 * k + 0] = sl[k].x; acc[4 * k + 1] = sl[k].y;
            acc[4 * k + 2] = sl[k].z; acc[4 * k + 3] = sl[k].w;
        }
#pragma unroll 8
        for (int c = 0; c < kDK; ++c) {
            const float a = Ms[m * kMsLd + c];
            const float4 *sr = (const float4 *)(Ss + c * kComposeCols + cb);
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const float4 x = sr[q];
                acc[4 * q + 0] = fmaf(a, x.x, acc[4 * q + 0]);
                acc[4 * q + 1] = fmaf(a, x.y, acc[4 * q + 1]);
                acc[4 * q + 2] = fmaf(a, x.z, acc[4 * q + 2]);
                acc[4 * q + 3] = fmaf(a, x.w, acc[4 * q + 3]);
            }
        }
        __syncthreads();             // every read of Ss and Ms is done
#pragma unroll
        for (int q = 0; q < 2; ++q)
            *(float4 *)(Ss + m * kComposeCols + cb + 4 * q) =
                make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
        __syncthreads();
    }
    if (Sf) {
        float4 *d = (float4 *)(Sf + ((size_t)n * H + h) * kStateF32 + (size_t)m * kDV + v0 + cb);
        const float4 *src = (const float4 *)(Ss + m * kComposeCols + cb);
#pragma unroll
        for (int q = 0; q < 2; ++q) d[q] = src[q];
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
    uint8_t *sm = align_smem_1024(smraw);
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
    }
    // While the operands arrive, every epilogue thread fetches its partial output
    // row (M = 64: TMEM lane 32 w + i holds row 16 w + i; lanes 16..31 have none).
    const int t0 = cu[n] + c * kChunk, len = min(kChunk, cu[n + 1] - t0);
    const int r = 16 * warp + lane;
    const bool has_row = lane < 16 && r < len;
    uint4 *orow = (uint4 *)(o + ((size_t)(t0 + (has_row ? r : 0)) * H + h) * kDV);
    uint4 ov[16];
    if (has_row) {
#pragma unroll
        for (int i = 0; i < 16; ++i) ov[i] = orow[i];
    }
    if (tid == 0) {
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
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t ra[32];
            tmem_ld32(tmem_addr(tb, 32 * warp, 32 * q), ra);
            tmem_ld_wait();
            if (has_row) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t *acc = ra + 8 * i;
                    uint4 &x = ov[4 * q + i];
                    uint32_t *w = &x.x;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(*(const __nv_bfloat162 *)&w[e]);
                        w[e] = pack_bf16(f.x + __uint_as_float(acc[2 * e]),
                                         f.y + __uint_as_float(acc[2 * e + 1]));
                    }
                }
            }
        }
        if (has_row) {
#pragma unroll
            for (int i = 0; i < 16; ++i) orow[i] = ov[i];
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, 128);
}

// ------------------------------------------------------------------ debug --

// Stage a1 on its own: G[t,h,c] = the inclusive cumulative gate of its 64-token
// chunk (chunks aligned to each sequence start), with the intra kernel's gate
// arithmetic.  One CTA of 128 threads (channels) per (chunk, head).
__global__ void __launch_bounds__(128)
debug_gate_kernel(const __nv_bfloat16 *__restrict__ z, const float *__restrict__ A,
                  const int2 *__restrict__ chunk_loc, const int32_t *__restrict__ chunk_off, int N,
                  int H, float *__restrict__ Gout)
{
    const int h = blockIdx.x % H, g = blockIdx.x / H;
    if (g >= chunk_off[N]) return;
    const int2 loc = chunk_loc[g];
    const int c = threadIdx.x;
    const float eAn = -ex2_approx(A[(size_t)h * kDK + c] * kLog2e) * kLog2e;
    float acc = 0.f;
    for (int r = 0; r < loc.y; ++r) {
        const size_t idx = ((size_t)(loc.x + r) * H + h) * kDK + c;
        acc += gate_fast(eAn, __bfloat162float(z[idx]));
        Gout[idx] = acc;
    }
}

// Stage a2's outputs read back from the per-(chunk, head) blocks: W (rows 0..63 of
// the [W; Qt] image) and U, as fp32 [T, H, 128].
__global__ void __launch_bounds__(256)
debug_unpack_kernel(const uint8_t *__restrict__ blocks, int64_t max_chunks,
                    const int2 *__restrict__ chunk_loc, const int32_t *__restrict__ chunk_off, int N,
                    int H, float *__restrict__ Wout, float *__restrict__ Uout)
{
    const int h = blockIdx.x % H, g = blockIdx.x / H;
    if (g >= chunk_off[N]) return;
    const int2 loc = chunk_loc[g];
    const uint8_t *blk = blocks + ((size_t)h * max_chunks + g) * kBlockBytes;
    for (int e = threadIdx.x; e < loc.y * kDK; e += 256) {
        const int r = e / kDK, c = e % kDK;
        const size_t idx = ((size_t)(loc.x + r) * H + h) * kDK + c;
        if (Wout)
            Wout[idx] = __bfloat162float(*(const __nv_bfloat16 *)(blk + kOffWQ + sw128_offset(r, c, 128)));
        if (Uout)
            Uout[idx] = __bfloat162float(*(const __nv_bfloat16 *)(blk + kOffU + u_offset(r, c)));
    }
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
// {64, 1, 64} box and the 128-byte swizzle: one K half of one chunk of one head
// per load, landing as the K-major operand image of 64 rows x 128 bytes.
bool encode_rows_map(CUtensorMap *map, const void *base, int32_t T, int32_t H)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)kDK, (cuuint64_t)H, (cuuint64_t)(T > 0 ? T : 1)};
    const cuuint64_t strides[2] = {(cuuint64_t)kDK * 2, (cuuint64_t)H * kDK * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)kChunk};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// o [T][H][128] bf16 as a 3-D tensor (channel, head, token) with a {128, 1, 64}
// box and no swizzle: one chunk's output rows of one head per TMA store, from
// a dense [64][128] staging tile.
bool encode_out_map(CUtensorMap *map, void *base, int32_t T, int32_t H)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)kDV, (cuuint64_t)H, (cuuint64_t)(T > 0 ? T : 1)};
    const cuuint64_t strides[2] = {(cuuint64_t)kDV * 2, (cuuint64_t)H * kDV * 2};
    const cuuint32_t box[3] = {(cuuint32_t)kDV, 1, (cuuint32_t)kChunk};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

namespace {

// SMs the split plan targets: the 148 of a B200.
constexpr int64_t kSplitSms = 148;
constexpr int64_t kMaxSegments = 16;

// Workspace layout: plan region (offsets, order, chunk table), per-(chunk, head)
// blocks, then (split only)
// Sx and Mx [N][G][H] fp32 states, S_in images [N][G][H] and E images [H][chunks].
struct WsLayout {
    size_t plan, loc, blocks, sx, mx, simg, eimg, pairs, total;
};

// With the unbounded gate the layout ends with the pair kernel's diagonal
// tiles: 8 KiB per (chunk, head).
WsLayout ws_layout(int32_t total_tokens, int32_t num_seqs, int32_t H, int G, int gate = kGateBounded)
{
    WsLayout w{};
    if (num_seqs <= 0) return w;
    const int64_t max_chunks = ((int64_t)total_tokens + 63LL * num_seqs) / kChunk;
    auto up = [](size_t x) { return (x + 1023) & ~(size_t)1023; };
    w.plan = 0;
    w.loc = ((size_t)(3 * num_seqs + 3) * sizeof(int32_t) + 7) & ~(size_t)7;
    w.blocks = up(w.loc + (size_t)max_chunks * sizeof(int2));
    size_t end = w.blocks + (size_t)H * max_chunks * kBlockBytes;
    if (G > 1) {
        const size_t states = (size_t)num_seqs * G * H;
        w.sx = up(end);
        w.mx = w.sx + states * kStateF32 * sizeof(float);
        w.simg = w.mx + states * kStateF32 * sizeof(float);
        w.eimg = w.simg + states * kSinImg;
        end = w.eimg + (size_t)H * max_chunks * kEImg;
    }
    if (gate == kGateSoftplus) {
        w.pairs = up(end);
        end = w.pairs + (size_t)H * max_chunks * 2048 * sizeof(float);
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

size_t tc_workspace_bytes(int32_t total_tokens, int32_t num_seqs, int32_t H, int segments, int gate)
{
    return ws_layout(total_tokens, num_seqs, H, segments, gate).total;
}

cudaError_t launch_prefill_tensor_core(const PrefillArgs &a, cudaStream_t stream)
{
    if (a.dk != kDK || a.dv != kDV || !a.bf16) return cudaErrorInvalidValue;
    const int G = a.segments > 1 ? a.segments : 1;
    if (G > 1 && a.ckpt_every > 0) return cudaErrorInvalidValue;
    const int64_t max_chunks = ((int64_t)a.total_tokens + 63LL * a.num_seqs) / kChunk;
    const bool softplus = a.gate == kGateSoftplus;
    const WsLayout w = ws_layout(a.total_tokens, a.num_seqs, a.H, G, a.gate);
    uint8_t *ws = (uint8_t *)a.workspace;
    int32_t *chunk_off = (int32_t *)ws;
    int32_t *ckpt_off = chunk_off + a.num_seqs + 1;
    int32_t *order = ckpt_off + a.num_seqs + 1;
    int2 *chunk_loc = (int2 *)(ws + w.loc);
    uint8_t *blocks = ws + w.blocks;
    float *Sx = G > 1 ? (float *)(ws + w.sx) : nullptr;
    float *Mx = G > 1 ? (float *)(ws + w.mx) : nullptr;
    uint8_t *Simg = G > 1 ? ws + w.simg : nullptr;
    uint8_t *Eimg = G > 1 ? ws + w.eimg : nullptr;
    cudaError_t err;

    auto intra_fn = softplus ? intra_kernel<kGateSoftplus> : intra_kernel<kGateBounded>;
    err = cudaFuncSetAttribute(intra_fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)(kISmem + 1024));
    if (err != cudaSuccess) return err;
    // Two intra CTAs share an SM: ask for the largest shared-memory carveout.
    err = cudaFuncSetAttribute(intra_fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                               (int)cudaSharedmemCarveoutMaxShared);
    if (err != cudaSuccess) return err;
    if (softplus) {
        err = cudaFuncSetAttribute(diag_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)kPairSmem);
        if (err != cudaSuccess) return err;
    }
    auto state_fn = a.dbg_delta ? state_kernel<true> : state_kernel<false>;
    err = cudaFuncSetAttribute(state_fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStateSmem);
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
                                                ckpt_off, order, chunk_loc);
    a.mark(1, stream);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;

    if (max_chunks > 0) {
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) == cudaSuccess)
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const int64_t items = max_chunks * a.H;
        const unsigned grid = (unsigned)(items < 2 * sms ? items : 2 * sms);
        CUtensorMap mk, mq, mv, mz;
        if (!encode_rows_map(&mk, a.k, a.total_tokens, a.H) || !encode_rows_map(&mq, a.q, a.total_tokens, a.H) ||
            !encode_rows_map(&mv, a.v, a.total_tokens, a.H) || !encode_rows_map(&mz, a.z, a.total_tokens, a.H))
            return cudaErrorInvalidValue;
        float *pairs = softplus ? (float *)(ws + w.pairs) : nullptr;
        if (softplus) {
            diag_pair_kernel<<<(unsigned)(max_chunks * a.H), kPairThreads, kPairSmem, stream>>>(
                (const __nv_bfloat16 *)a.k, (const __nv_bfloat16 *)a.q, (const __nv_bfloat16 *)a.z,
                a.A, chunk_loc, chunk_off, a.num_seqs, a.H, max_chunks, pairs);
            if ((err = cudaGetLastError()) != cudaSuccess) return err;
        }
        intra_fn<<<grid, kIntraThreads, kISmem + 1024, stream>>>(
            mk, mq, mv, mz, a.A, a.beta, chunk_loc, chunk_off, a.num_seqs, a.H,
            blocks, max_chunks, a.status, pairs);
        err = cudaGetLastError();
        if (err != cudaSuccess) return err;
    }
    a.mark(2, stream);
    CUtensorMap mo;
    memset(&mo, 0, sizeof(mo));  // with no tokens (o may be null) no chunk stores anything
    if (a.total_tokens > 0 && !encode_out_map(&mo, a.o, a.total_tokens, a.H))
        return cudaErrorInvalidValue;
    state_fn<<<(unsigned)((int64_t)a.num_seqs * a.H * (2 * G - 1)), kStateThreads, kStateSmem,
               stream>>>(
        mo, a.cu_seqlens, chunk_off, order, a.num_seqs, a.H, blocks, max_chunks, a.initial_state,
        a.final_state, (__nv_bfloat16 *)a.o, a.status, a.ckpt_every, ckpt_off, a.checkpoints,
        G, Sx, Mx, Eimg, a.dbg_delta);
    a.mark(3, stream);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    if (max_chunks > 0 && a.dbg_G) {
        debug_gate_kernel<<<(unsigned)(max_chunks * a.H), 128, 0, stream>>>(
            (const __nv_bfloat16 *)a.z, a.A, chunk_loc, chunk_off, a.num_seqs, a.H, a.dbg_G);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    if (max_chunks > 0 && (a.dbg_W || a.dbg_U)) {
        debug_unpack_kernel<<<(unsigned)(max_chunks * a.H), 256, 0, stream>>>(
            blocks, max_chunks, chunk_loc, chunk_off, a.num_seqs, a.H, a.dbg_W, a.dbg_U);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    if (G == 1) return cudaSuccess;

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
