// Backward pass of exact attention with recomputation on the fifth-generation
// tensor cores: dQ, dK, dV from Q, K, V, O, dO and the forward's log-sum-exp,
// without the n x n weight matrix in memory ("Sviluppo AI ed Algebra Lineare", section
// "Ricalcolo nel Backward Pass (Recomputation)": only the row statistics are
// kept, and the score and weight blocks are recomputed tile by tile on chip).
// For one query head and its kept keys:
//
//   P_ij  = exp(scale q_i.k_j - LSE_i)        (the forward's LSE normalises P)
//   dV_j += sum_i P_ij dO_i
//   dS_ij = P_ij (dO_i.v_j - dO_i.O_i)        (sum_k P_ik dP_ik = dO_i.O_i)
//   dQ_i  = scale sum_j dS_ij k_j
//   dK_j += scale sum_i dS_ij q_i              (dK, dV summed over the group's query heads)
//
// Three kernels, all deterministic (fixed summation order, no atomics):
//
// bwd_prep_kernel: one warp per query row writes dO.O and LSE * log2(e) into a
// workspace padded to a multiple of 64 rows per head (pad rows: weight 0, dS 0).
//
// bwd_dkdv_tc: one CTA per (128-key block, kv head, batch row).  K and V stay in
// shared memory; the query blocks (64 rows) of every query head of the group
// stream through a shared-memory ring.  Per block t:
//   S^T = K Q^T, dP^T = V dO^T      SS MMAs, M = 128 keys, N = 64 queries, into one
//                                   of two TMEM buffers (double-buffered)
//   softmax warps (thread = key row): P^T = exp2(S^T c - L_i), dS^T = P^T (dP^T - D_i),
//                                   both rounded to bf16 and stored back into TMEM
//                                   over their own fp32 columns
//   dV += P^T dO, dK += dS^T Q      TS MMAs (A from TMEM, B = the dO / Q tile read
//                                   MN-major), accumulators in TMEM for the whole CTA
// The MMA warp issues S^T/dP^T of block t + 1 before dV/dK of block t, so the
// tensor core works on the next block while the softmax warps finish this one.
//
// bwd_dq_tc: one CTA per (128-query block, head, batch row); the key blocks (64
// rows) stream through the ring: S = Q K^T, dP = dO V^T (SS), dS in the softmax
// warps (thread = query row), dQ += dS K (TS, K read MN-major).  Splitting dQ from
// dK/dV recomputes S and dP once more (7 products instead of 5) in exchange for no
// atomics and no cross-CTA reduction.
//
// Warps 0-3: softmax and epilogue (TMEM lanes 0-127); warp 4: TMA producer;
// warp 5: TMEM allocation and MMA issue (lane 0 issues).  Masked entries get the
// exponent -inf (weight exactly 0) through a select, never a branch around the
// exponential.  Every mbarrier wait is bounded; a wait that gives up records its
// site, the CTA's roles stop, copies and MMAs in flight are drained (bounded) and
// TMEM is freed before the CTA returns.
#include <algorithm>
#include <cmath>
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace attn {
namespace {

using namespace dev;

constexpr int kBig = 128;    // rows of the resident tiles (keys in dK/dV, queries in dQ)
constexpr int kStep = 64;    // rows of the streamed tiles
constexpr int kThreads = 192;
constexpr int kProducerWarp = 4, kMmaWarp = 5;
constexpr int kTmemCols = 512;
constexpr int kRing = 3;     // shared-memory stages of the streamed tiles
constexpr float kLog2e = 1.4426950408889634f;

enum : uint32_t {
    kSiteTcRes = 0x41, kSiteTcQFull = 0x42, kSiteTcQEmpty = 0x43, kSiteTcSFull = 0x44, kSiteTcP = 0x45,
    kSiteTcAcc = 0x46
};

__global__ void bwd_prep_kernel(const BwdArgs a) {
    const long long rows = (long long)a.B * a.H * a.n_q_pad;
    const int lane = threadIdx.x % 32;
    const long long warp0 = (blockIdx.x * (long long)blockDim.x + threadIdx.x) / 32;
    const long long nwarps = (long long)gridDim.x * blockDim.x / 32;
    for (long long r = warp0; r < rows; r += nwarps) {
        const long long bh = r / a.n_q_pad;
        const int i = (int)(r % a.n_q_pad);
        float dd = 0.f, l2 = INFINITY;   // pad rows: weight exp2(x - inf) = 0 and dS = 0
        if (i < a.n_q) {
            const long long base = (bh * a.n_q + i) * a.d;
            const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(a.o) + base / 2;
            const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(a.d_o) + base / 2;
            for (int c = lane; c < a.d / 2; c += 32) {
                const float2 x = __bfloat1622float2(o2[c]);
                const float2 y = __bfloat1622float2(g2[c]);
                dd = fmaf(x.x, y.x, fmaf(x.y, y.y, dd));
            }
#pragma unroll
            for (int s = 16; s > 0; s >>= 1) dd += __shfl_xor_sync(0xffffffffu, dd, s);
            const float lse = a.lse[bh * a.n_q + i];
            l2 = lse == -INFINITY ? INFINITY : lse * kLog2e;   // a row with no kept key: every weight 0
        }
        if (lane == 0) {
            a.ws_dd[r] = dd;
            a.ws_l2[r] = l2;
        }
    }
}

// A [rows][D] bf16 tile as TMA writes it: D/64 column groups of [rows][128 bytes],
// 128-byte swizzle; filled by boxes of 64 rows x 64 columns.
template <int D, int R>
struct Tile {
    static constexpr int kGroupBytes = R * 128;
    static constexpr int kBytes = (D / 64) * kGroupBytes;
};

template <int D, int R>
__device__ __forceinline__ void tma_tile(uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int row0, int head,
                                         int batch) {
#pragma unroll
    for (int g = 0; g < D / 64; ++g)
#pragma unroll
        for (int r = 0; r < R / 64; ++r)
            tma_load_4d(dst + g * Tile<D, R>::kGroupBytes + r * 64 * 128, map, bar, g * 64, row0 + 64 * r, head,
                        batch);
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// D (+)= A B^T over K = D columns, both operands K-major tiles (A: 128 rows, B: 64 rows).
template <int D>
__device__ __forceinline__ void mma_ss_rows(bool leader, uint32_t d_tmem, uint32_t sa, uint32_t sb) {
    constexpr uint32_t idesc = idesc_bf16_f32(kBig, kStep, 0, 0);
    const uint64_t a0 = smem_desc_sw128(sa, 16, 1024), b0 = smem_desc_sw128(sb, 16, 1024);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        // 16 columns = 32 bytes inside a 128-byte row; column groups of 64 are a whole
        // [rows][128 B] group apart
        const uint64_t oa = (uint64_t)((kk & 3) * 2 + (kk >> 2) * (Tile<D, kBig>::kGroupBytes >> 4));
        const uint64_t ob = (uint64_t)((kk & 3) * 2 + (kk >> 2) * (Tile<D, kStep>::kGroupBytes >> 4));
        mma_bf16_ss(leader, d_tmem, a0 + oa, b0 + ob, idesc, kk > 0 ? 1u : 0u);
    }
}

// D (+)= A B with A = 128 x 64 bf16 in TMEM (2 values per column) and B = a
// 64-row tile read MN-major (K = its rows, N = its D columns).
template <int D>
__device__ __forceinline__ void mma_ts_cols(bool leader, uint32_t d_tmem, uint32_t a_tmem, uint32_t sb,
                                            bool accumulate) {
    constexpr uint32_t idesc = idesc_bf16_f32(kBig, D, 0, 1);
    const uint64_t b0 = smem_desc_sw128(sb, Tile<D, kStep>::kGroupBytes, 1024);
#pragma unroll
    for (int kk = 0; kk < kStep / 16; ++kk)  // 16 rows of B = 2 KB per step
        mma_bf16_ts(leader, d_tmem, a_tmem + kk * 8, b0 + (uint64_t)(kk * 128), idesc,
                    (accumulate || kk > 0) ? 1u : 0u);
}

template <int N>
__device__ __forceinline__ void pin(uint32_t (&r)[N]) {
#pragma unroll
    for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

// Write 32 fp32 accumulator columns of this thread's row as bf16 (times mul) to dst.
__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const uint32_t (&r)[32], float mul) {
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * mul, __uint_as_float(r[2 * i + 1]) * mul);
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) d4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
}

// dK/dV softmax of one key row over 64 query columns: P^T = exp2(S^T c - L_col) and
// dS^T = P^T (dP^T - D_col), packed to bf16 pairs.  kMasked: columns col < lim dropped.
template <bool kMasked>
__device__ __forceinline__ void weights_dkdv(const uint32_t (&s)[64], const uint32_t (&dp)[64], const float4* l2,
                                             const float4* dd, float c, int lim, uint32_t (&pw)[32],
                                             uint32_t (&dw)[32]) {
#pragma unroll
    for (int q = 0; q < 16; ++q) {
        const float4 L = l2[q], Dd = dd[q];
        const float lv[4] = {L.x, L.y, L.z, L.w}, dv[4] = {Dd.x, Dd.y, Dd.z, Dd.w};
        float p[4], d[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int col = 4 * q + e;
            float x = fmaf(__uint_as_float(s[col]), c, -lv[e]);
            if (kMasked) x = col >= lim ? x : -INFINITY;
            p[e] = ex2_approx(x);
            d[e] = p[e] * (__uint_as_float(dp[col]) - dv[e]);
        }
        pw[2 * q] = pack_bf16x2(p[0], p[1]);
        pw[2 * q + 1] = pack_bf16x2(p[2], p[3]);
        dw[2 * q] = pack_bf16x2(d[0], d[1]);
        dw[2 * q + 1] = pack_bf16x2(d[2], d[3]);
    }
}

// dQ softmax of one query row over 64 key columns: dS = exp2(S c - L) (dP - D), packed
// to bf16 pairs.  kMasked: columns past lim or with a cleared flag byte dropped.
template <bool kMasked>
__device__ __forceinline__ void weights_dq(const uint32_t (&s)[64], const uint32_t (&dp)[64],
                                           const uint32_t* keep_w, float c, float l2, float ddi, int lim,
                                           uint32_t (&dw)[32]) {
#pragma unroll
    for (int q = 0; q < 16; ++q) {
        const uint32_t kw = kMasked ? keep_w[q] : 0xffffffffu;
        float d[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int col = 4 * q + e;
            float x = fmaf(__uint_as_float(s[col]), c, -l2);
            if (kMasked) x = (col <= lim && ((kw >> (8 * e)) & 0xffu) != 0u) ? x : -INFINITY;
            d[e] = ex2_approx(x) * (__uint_as_float(dp[col]) - ddi);
        }
        dw[2 * q] = pack_bf16x2(d[0], d[1]);
        dw[2 * q + 1] = pack_bf16x2(d[2], d[3]);
    }
}

struct TcBars {
    uint64_t res_full;      // resident tiles (K, V or Q, dO)
    uint64_t full[kRing], empty[kRing];   // streamed stages
    uint64_t s_full[2];     // S and dP of a stage computed
    uint64_t p_ready[2];    // P / dS of a stage in TMEM (128 arrivals)
    uint64_t acc_full;      // last accumulating MMA done
    uint64_t fin;           // abort path: every MMA issued so far done
    uint32_t tmem_base;
    int abort_flag;
};

template <int D>
struct DkdvTcSmem {
    static constexpr int kBigT = Tile<D, kBig>::kBytes, kStepT = Tile<D, kStep>::kBytes;
    static constexpr int kOffK = 0, kOffV = kBigT, kOffQ = 2 * kBigT, kOffO = 2 * kBigT + kRing * kStepT;
    static constexpr int kOffL = 2 * kBigT + 2 * kRing * kStepT;   // float l2[kRing][64], dd[kRing][64]
    static constexpr int kOffBar = kOffL + 2 * kRing * kStep * 4;
    static constexpr int kBytes = kOffBar + (int)sizeof(TcBars);
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo, const BwdArgs a,
                unsigned int* status) {
    using L = DkdvTcSmem<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float* s_l2 = reinterpret_cast<float*>(smem + L::kOffL);   // [kRing][64]
    float* s_dd = s_l2 + kRing * kStep;                        // [kRing][64]
    TcBars& bar = *reinterpret_cast<TcBars*>(smem + L::kOffBar);
    volatile int* ab = &bar.abort_flag;

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int n_kb = (a.n_kv + kBig - 1) / kBig;
    const int per = a.H_kv * a.B;
    const int kb = blockIdx.x / per;   // the first key blocks are the heaviest under a causal mask: first
    const int g = (blockIdx.x % per) % a.H_kv, b = (blockIdx.x % per) / a.H_kv;
    if (kb >= n_kb) return;
    const int j0 = kb * kBig;
    const int group = a.H / a.H_kv;
    const int off = a.n_kv - a.n_q;    // causal: key j is visible to query i when j <= i + off
    const int n_qb = (a.n_q + kStep - 1) / kStep;
    const int qb0 = a.causal ? max(0, j0 - off) / kStep : 0;
    const int per_head = n_qb - qb0;
    const int steps = group * per_head;   // >= 1: row n_q - 1 sees every key when causal

    if (tid == 0) {
        mbar_init(&bar.res_full, 1);
        for (int s = 0; s < kRing; ++s) {
            mbar_init(&bar.full[s], 1);
            mbar_init(&bar.empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar.s_full[s], 1);
            mbar_init(&bar.p_ready[s], 128);
        }
        mbar_init(&bar.acc_full, 1);
        mbar_init(&bar.fin, 1);
        bar.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&bar.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar.tmem_base;
    constexpr uint32_t kColDV = 0, kColDK = D;
    auto colS = [](int st) { return (uint32_t)(2 * D + st * kStep); };
    auto colP = [](int st) { return (uint32_t)(2 * D + 2 * kStep + st * kStep); };   // dP^T, then dS^T

    if (warp == kProducerWarp) {
        if (lane == 0) {
            int issued = 0;
            bool ok = true;
            mbar_arrive_expect_tx(&bar.res_full, 2 * L::kBigT);
            tma_tile<D, kBig>(smem + L::kOffK, &tk, &bar.res_full, j0, g, b);
            tma_tile<D, kBig>(smem + L::kOffV, &tv, &bar.res_full, j0, g, b);
            for (int t = 0; t < steps; ++t) {
                const int st = t % kRing;
                if (!mbar_wait(&bar.empty[st], ((t / kRing) & 1) ^ 1, ab, status, kSiteTcQEmpty)) {
                    ok = false;
                    break;
                }
                const int h = g * group + t / per_head, qb = qb0 + t % per_head;
                mbar_arrive_expect_tx(&bar.full[st], 2 * L::kStepT + 2 * kStep * 4);
                tma_tile<D, kStep>(smem + L::kOffQ + st * L::kStepT, &tq, &bar.full[st], qb * kStep, h, b);
                tma_tile<D, kStep>(smem + L::kOffO + st * L::kStepT, &tdo, &bar.full[st], qb * kStep, h, b);
                const size_t row0 = ((size_t)b * a.H + h) * a.n_q_pad + (size_t)qb * kStep;
                bulk_load(s_l2 + st * kStep, a.ws_l2 + row0, kStep * 4, &bar.full[st]);
                bulk_load(s_dd + st * kStep, a.ws_dd + row0, kStep * 4, &bar.full[st]);
                issued = t + 1;
            }
            if (!ok || *ab) {
                mbar_drain(&bar.res_full, 0);
                for (int t = max(0, issued - kRing); t < issued; ++t)
                    mbar_drain(&bar.full[t % kRing], (t / kRing) & 1);
            }
        }
    } else if (warp == kMmaWarp) {
        const bool leader = lane == 0;
        const uint32_t sK = smem_u32(smem + L::kOffK), sV = smem_u32(smem + L::kOffV);
        bool ok = warp_wait(&bar.res_full, 0, ab, status, kSiteTcRes);
        int t = 0;
        for (; ok && t <= steps; ++t) {
            if (t < steps) {
                const int st = t % kRing, tb = t & 1;
                ok = warp_wait(&bar.full[st], (t / kRing) & 1, ab, status, kSiteTcQFull);
                if (!ok) break;
                tc_fence_after();
                const uint32_t sQ = smem_u32(smem + L::kOffQ + st * L::kStepT);
                const uint32_t sO = smem_u32(smem + L::kOffO + st * L::kStepT);
                mma_ss_rows<D>(leader, tmem + colS(tb), sK, sQ);   // S^T = K Q^T
                mma_ss_rows<D>(leader, tmem + colP(tb), sV, sO);   // dP^T = V dO^T
                mma_commit(leader, &bar.s_full[tb]);
            }
            if (t >= 1) {
                const int u = t - 1, su = u % kRing, ub = u & 1;
                ok = warp_wait(&bar.p_ready[ub], (u >> 1) & 1, ab, status, kSiteTcP);
                if (!ok) break;
                tc_fence_after();
                const uint32_t sQ = smem_u32(smem + L::kOffQ + su * L::kStepT);
                const uint32_t sO = smem_u32(smem + L::kOffO + su * L::kStepT);
                mma_ts_cols<D>(leader, tmem + kColDV, tmem + colS(ub), sO, u > 0);   // dV += P^T dO
                mma_ts_cols<D>(leader, tmem + kColDK, tmem + colP(ub), sQ, u > 0);   // dK += dS^T Q
                mma_commit(leader, &bar.empty[su]);
                if (u == steps - 1) mma_commit(leader, &bar.acc_full);
            }
        }
        if (!ok) {
            mma_commit(leader, &bar.fin);
            if (leader) mbar_drain(&bar.fin, 0);
        }
        __syncwarp();
    } else {
        // softmax warps: thread = key row j0 + tid (TMEM lane tid)
        const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
        const int j = j0 + tid;
        const bool key_ok = j < a.n_kv && (a.key_mask == nullptr || a.key_mask[(size_t)b * a.n_kv + j] != 0);
        const float c = a.scale * kLog2e;
        bool ok = true;
        for (int t = 0; t < steps; ++t) {
            const int st = t % kRing, tb = t & 1;
            // full[st] (already complete) makes the stage's copied rows visible to this thread
            ok = mbar_wait(&bar.s_full[tb], (t >> 1) & 1, ab, status, kSiteTcSFull) &&
                 mbar_wait(&bar.full[st], (t / kRing) & 1, ab, status, kSiteTcQFull);
            if (!__all_sync(0xffffffffu, ok)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int i0 = (qb0 + t % per_head) * kStep;
            const bool diag = a.causal && (j0 + kBig - 1 > i0 + off);
            uint32_t s[64], dp[64];
            tmem_ld32(tmem + lane_off + colS(tb), s);
            tmem_ld32(tmem + lane_off + colS(tb) + 32, s + 32);
            tmem_ld32(tmem + lane_off + colP(tb), dp);
            tmem_ld32(tmem + lane_off + colP(tb) + 32, dp + 32);
            tmem_wait_ld();
            pin(s);
            pin(dp);
            // query column col is kept iff col >= lim (a masked key row keeps none); the
            // exponent of a dropped entry is -inf, so its weight is exactly 0 with no branch
            const int lim = !key_ok ? kStep : (diag ? j - off - i0 : 0);
            const float4* l2 = reinterpret_cast<const float4*>(s_l2 + st * kStep);
            const float4* dd = reinterpret_cast<const float4*>(s_dd + st * kStep);
            uint32_t pw[32], dw[32];
            if (__all_sync(0xffffffffu, lim <= 0))
                weights_dkdv<false>(s, dp, l2, dd, c, 0, pw, dw);
            else
                weights_dkdv<true>(s, dp, l2, dd, c, lim, pw, dw);
            tmem_st32(tmem + lane_off + colS(tb), pw);
            tmem_st32(tmem + lane_off + colP(tb), dw);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bar.p_ready[tb]);
        }
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bar.acc_full, 0, ab, status, kSiteTcAcc));
        if (ok) {
            tc_fence_after();
            __nv_bfloat16* dk_row = static_cast<__nv_bfloat16*>(a.dk) + (((size_t)b * a.H_kv + g) * a.n_kv + j) * D;
            __nv_bfloat16* dv_row = static_cast<__nv_bfloat16*>(a.dv) + (((size_t)b * a.H_kv + g) * a.n_kv + j) * D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t r[32];
                tmem_ld32(tmem + lane_off + kColDV + c0, r);
                tmem_wait_ld();
                pin(r);
                if (j < a.n_kv) store_row32(dv_row + c0, r, 1.f);
                tmem_ld32(tmem + lane_off + kColDK + c0, r);
                tmem_wait_ld();
                pin(r);
                if (j < a.n_kv) store_row32(dk_row + c0, r, a.scale);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int D>
struct DqTcSmem {
    static constexpr int kBigT = Tile<D, kBig>::kBytes, kStepT = Tile<D, kStep>::kBytes;
    static constexpr int kOffQ = 0, kOffO = kBigT, kOffK = 2 * kBigT, kOffV = 2 * kBigT + kRing * kStepT;
    static constexpr int kOffKeep = 2 * kBigT + 2 * kRing * kStepT;   // uint8 keep[kRing][64]
    static constexpr int kOffBar = kOffKeep + kRing * kStep;
    static constexpr int kBytes = kOffBar + (int)sizeof(TcBars);
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
              const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo, const BwdArgs a,
              unsigned int* status) {
    using L = DqTcSmem<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* s_keep = smem + L::kOffKeep;   // [kRing][64]
    TcBars& bar = *reinterpret_cast<TcBars*>(smem + L::kOffBar);
    volatile int* ab = &bar.abort_flag;

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int n_qb = (a.n_q + kBig - 1) / kBig;
    const int per = a.H * a.B;
    const int qb = n_qb - 1 - (int)(blockIdx.x / per);   // the last query blocks are the heaviest: first
    const int h = (blockIdx.x % per) % a.H, b = (blockIdx.x % per) / a.H;
    if (qb < 0) return;
    const int g = h / (a.H / a.H_kv);
    const int q0 = qb * kBig;
    const int off = a.n_kv - a.n_q;
    const int n_kb_all = (a.n_kv + kStep - 1) / kStep;
    int n_kb = n_kb_all;
    if (a.causal) {
        const int j_max = min(q0 + kBig, a.n_q) - 1 + off;   // last key a row of this block sees
        n_kb = j_max < 0 ? 0 : min(n_kb_all, j_max / kStep + 1);
    }

    if (tid == 0) {
        mbar_init(&bar.res_full, 1);
        for (int s = 0; s < kRing; ++s) {
            mbar_init(&bar.full[s], 1);
            mbar_init(&bar.empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar.s_full[s], 1);
            mbar_init(&bar.p_ready[s], 128);
        }
        mbar_init(&bar.acc_full, 1);
        mbar_init(&bar.fin, 1);
        bar.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&bar.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar.tmem_base;
    constexpr uint32_t kColDQ = 0;
    auto colS = [](int st) { return (uint32_t)(D + st * kStep); };
    auto colP = [](int st) { return (uint32_t)(D + 2 * kStep + st * kStep); };   // dP, then dS

    if (warp == kProducerWarp) {
        int issued = 0;
        bool ok = true;
        if (lane == 0 && n_kb > 0) {
            mbar_arrive_expect_tx(&bar.res_full, 2 * L::kBigT);
            tma_tile<D, kBig>(smem + L::kOffQ, &tq, &bar.res_full, q0, h, b);
            tma_tile<D, kBig>(smem + L::kOffO, &tdo, &bar.res_full, q0, h, b);
        }
        for (int t = 0; t < n_kb; ++t) {
            const int st = t % kRing;
            ok = warp_wait(&bar.empty[st], ((t / kRing) & 1) ^ 1, ab, status, kSiteTcQEmpty);
            if (!ok) break;
            // key flags of the block (plain stores, published by lane 0's arrive below)
            for (int r = lane; r < kStep; r += 32) {
                const int jj = t * kStep + r;
                s_keep[st * kStep + r] =
                    jj < a.n_kv && (a.key_mask == nullptr || a.key_mask[(size_t)b * a.n_kv + jj] != 0);
            }
            __threadfence_block();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive_expect_tx(&bar.full[st], 2 * L::kStepT);
                tma_tile<D, kStep>(smem + L::kOffK + st * L::kStepT, &tk, &bar.full[st], t * kStep, g, b);
                tma_tile<D, kStep>(smem + L::kOffV + st * L::kStepT, &tv, &bar.full[st], t * kStep, g, b);
            }
            issued = t + 1;
        }
        if (lane == 0 && (!ok || *ab)) {
            if (n_kb > 0) mbar_drain(&bar.res_full, 0);
            for (int t = max(0, issued - kRing); t < issued; ++t) mbar_drain(&bar.full[t % kRing], (t / kRing) & 1);
        }
    } else if (warp == kMmaWarp) {
        const bool leader = lane == 0;
        const uint32_t sQ = smem_u32(smem + L::kOffQ), sO = smem_u32(smem + L::kOffO);
        bool ok = n_kb == 0 || warp_wait(&bar.res_full, 0, ab, status, kSiteTcRes);
        for (int t = 0; ok && t <= n_kb && n_kb > 0; ++t) {
            if (t < n_kb) {
                const int st = t % kRing, tb = t & 1;
                ok = warp_wait(&bar.full[st], (t / kRing) & 1, ab, status, kSiteTcQFull);
                if (!ok) break;
                tc_fence_after();
                const uint32_t sK = smem_u32(smem + L::kOffK + st * L::kStepT);
                const uint32_t sV = smem_u32(smem + L::kOffV + st * L::kStepT);
                mma_ss_rows<D>(leader, tmem + colS(tb), sQ, sK);   // S = Q K^T
                mma_ss_rows<D>(leader, tmem + colP(tb), sO, sV);   // dP = dO V^T
                mma_commit(leader, &bar.s_full[tb]);
            }
            if (t >= 1) {
                const int u = t - 1, su = u % kRing, ub = u & 1;
                ok = warp_wait(&bar.p_ready[ub], (u >> 1) & 1, ab, status, kSiteTcP);
                if (!ok) break;
                tc_fence_after();
                const uint32_t sK = smem_u32(smem + L::kOffK + su * L::kStepT);
                mma_ts_cols<D>(leader, tmem + kColDQ, tmem + colP(ub), sK, u > 0);   // dQ += dS K
                mma_commit(leader, &bar.empty[su]);
                if (u == n_kb - 1) mma_commit(leader, &bar.acc_full);
            }
        }
        if (!ok) {
            mma_commit(leader, &bar.fin);
            if (leader) mbar_drain(&bar.fin, 0);
        }
        __syncwarp();
    } else {
        // softmax warps: thread = query row q0 + tid (TMEM lane tid)
        const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
        const int i = q0 + tid;
        const size_t lrow = ((size_t)b * a.H + h) * a.n_q_pad + i;
        const bool row_in = i < a.n_q;
        const float l2 = row_in ? a.ws_l2[lrow] : INFINITY;   // rows past n_q: weight 0
        const float ddi = row_in ? a.ws_dd[lrow] : 0.f;
        const float c = a.scale * kLog2e;
        bool ok = true;
        for (int t = 0; t < n_kb; ++t) {
            const int st = t % kRing, tb = t & 1;
            // full[st] (already complete) makes the stage's copied rows visible to this thread
            ok = mbar_wait(&bar.s_full[tb], (t >> 1) & 1, ab, status, kSiteTcSFull) &&
                 mbar_wait(&bar.full[st], (t / kRing) & 1, ab, status, kSiteTcQFull);
            if (!__all_sync(0xffffffffu, ok)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int j0 = t * kStep;
            const bool diag = a.causal && (j0 + kStep - 1 > q0 + off);
            uint32_t s[64], dp[64];
            tmem_ld32(tmem + lane_off + colS(tb), s);
            tmem_ld32(tmem + lane_off + colS(tb) + 32, s + 32);
            tmem_ld32(tmem + lane_off + colP(tb), dp);
            tmem_ld32(tmem + lane_off + colP(tb) + 32, dp + 32);
            tmem_wait_ld();
            pin(s);
            pin(dp);
            // key column col is kept iff col <= lim and its flag is set (a key mask or the
            // end of the keys clears flags); dropped entries get exponent -inf, weight 0
            const int lim = diag ? i + off - j0 : kStep;
            const uint32_t* keep_w = reinterpret_cast<const uint32_t*>(s_keep + st * kStep);
            const bool flags_all = (a.key_mask == nullptr) && (j0 + kStep <= a.n_kv);
            uint32_t dw[32];
            if (flags_all && __all_sync(0xffffffffu, lim >= kStep - 1))
                weights_dq<false>(s, dp, keep_w, c, l2, ddi, kStep, dw);
            else
                weights_dq<true>(s, dp, keep_w, c, l2, ddi, lim, dw);
            tmem_st32(tmem + lane_off + colP(tb), dw);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bar.p_ready[tb]);
        }
        if (ok && n_kb > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bar.acc_full, 0, ab, status, kSiteTcAcc));
        if (ok) {
            __nv_bfloat16* dq_row = static_cast<__nv_bfloat16*>(a.dq) + (((size_t)b * a.H + h) * a.n_q + i) * D;
            if (n_kb == 0) {
                if (row_in) {
                    uint4* d4 = reinterpret_cast<uint4*>(dq_row);
                    for (int k = 0; k < D / 8; ++k) d4[k] = make_uint4(0u, 0u, 0u, 0u);
                }
            } else {
                tc_fence_after();
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_off + kColDQ + c0, r);
                    tmem_wait_ld();
                    pin(r);
                    if (row_in) store_row32(dq_row + c0, r, a.scale);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int D>
cudaError_t launch_tc_d(const BwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                        const CUtensorMap& tdo, unsigned int* status, cudaStream_t stream) {
    // more than half of an SM's shared memory: one CTA per SM, so the 512-column
    // TMEM allocation never waits for another CTA
    const int smem_kv = std::max(DkdvTcSmem<D>::kBytes + 1024, 118 * 1024);
    const int smem_q = std::max(DqTcSmem<D>::kBytes + 1024, 118 * 1024);
    cudaError_t e = cudaFuncSetAttribute(bwd_dkdv_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_kv);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bwd_dq_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_q);
    if (e != cudaSuccess) return e;
    const long long grid_kv = (long long)((a.n_kv + kBig - 1) / kBig) * a.H_kv * a.B;
    const long long grid_q = (long long)((a.n_q + kBig - 1) / kBig) * a.H * a.B;
    if (grid_kv > 0x7fffffffll || grid_q > 0x7fffffffll) return cudaErrorInvalidConfiguration;
    bwd_dkdv_tc<D><<<(unsigned)grid_kv, kThreads, smem_kv, stream>>>(tq, tk, tv, tdo, a, status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    bwd_dq_tc<D><<<(unsigned)grid_q, kThreads, smem_q, stream>>>(tq, tk, tv, tdo, a, status);
    return cudaGetLastError();
}

cudaError_t launch_bwd_tc(const BwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const CUtensorMap& tdo, unsigned int* status, cudaStream_t stream) {
    return a.d == 64 ? launch_tc_d<64>(a, tq, tk, tv, tdo, status, stream)
                     : launch_tc_d<128>(a, tq, tk, tv, tdo, status, stream);
}

}  // namespace

cudaError_t launch_bwd(const BwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, unsigned int* status, cudaStream_t stream) {
    const long long rows = (long long)a.B * a.H * a.n_q_pad;
    const long long blocks = std::min<long long>((rows + 7) / 8, 148ll * 16);
    bwd_prep_kernel<<<(unsigned)std::max<long long>(blocks, 1), 256, 0, stream>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_bwd_tc(a, tq, tk, tv, tdo, status, stream);
}

}  // namespace attn
