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
// workspace padded to a multiple of 128 rows per head (pad rows: weight 0, dS 0).
//
// bwd_dkdv_tc: one CTA per (128-key block, kv head, batch row).  K and V stay in
// shared memory; the 128-row query tiles of every query head of the group stream
// through two rings (Q: 3 stages, dO: 2 stages).  Per query tile t:
//   S^T = K Q^T, dP^T = V dO^T      SS MMAs, M = 128 keys, N = 128 queries
//   softmax warps (thread = key row): P^T = exp2(S^T c - L_i), dS^T = P^T (dP^T - D_i),
//                                   rounded to bf16 and stored into TMEM over the dP^T
//                                   columns they were computed from, in two halves of
//                                   64 queries, each announced on its own barrier
//   dV += P^T dO, dK += dS^T Q      TS MMAs (A from TMEM, B = the dO / Q rows of that
//                                   half, read MN-major), one pair per half
// bwd_dq_tc: one CTA per (128-query block, head, batch row); the 128-key K and V
// tiles stream through the rings: S = Q K^T, dP = dO V^T (SS), dS in the softmax
// warps (thread = query row), dQ += dS K (TS, K read MN-major), again in halves.
// Its TMEM (dQ, S, dP) leaves room for a second S buffer, so S_{t+1} is issued right
// after dP_t instead of waiting for the softmax warps to pick up S_t.
// Splitting dQ from dK/dV recomputes S and dP once more (7 products instead of 5)
// in exchange for no atomics and no cross-CTA reduction.
//
// Why 128-row streamed tiles: a tcgen05.mma of M = 128 costs about the same time
// for every N up to 128 (on B200, about 70 cycles per K = 16 step), so N = 64
// score products run at half the tensor rate.  With N = 128 the score and its
// gradient take 256 TMEM columns, which leaves no room for a second buffer beside
// the 256 accumulator columns (dK and dV).  The MMA order per tile t is therefore
//   S_{t+1} | dV, dK (first half of t) | dV, dK (second half of t) | dP_{t+1}
// where S_{t+1} starts as soon as the softmax warps have loaded S_t into registers,
// the first-half products run while the softmax warps compute the second half, and
// dP_{t+1} overwrites the P / dS columns only after the products that read them
// (tcgen05 MMAs of one CTA execute in issue order).  The softmax of a half takes
// about as long as the products that overlap it, so the tensor pipe stays busy.
//
// Warps 0-7: softmax and epilogue; warp w reads TMEM lanes 32 (w % 4) .. + 31 and
// columns 32 (w / 4) .. + 31 of each half.  Warp 8: TMA producer of the resident
// tiles and the first ring; warp 9: TMEM allocation and MMA issue (lane 0 issues);
// warp 10: TMA producer of the second ring.  Masked entries get the exponent -inf
// (weight exactly 0) through a select, never a branch around the exponential.
// Every mbarrier wait is bounded; a wait that gives up records its site, the CTA's
// roles stop, copies and MMAs in flight are drained (bounded) and TMEM is freed
// before the CTA returns.
#include <algorithm>
#include <cmath>
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace attn {
namespace {

using namespace dev;

constexpr int kBig = 128;      // rows of the resident tiles (keys in dK/dV, queries in dQ)
constexpr int kStep = 128;     // rows of the streamed tiles
constexpr int kHalf = 64;      // P / dS columns handed to the MMA warp at a time
constexpr int kThreads = 352;  // 8 softmax warps, producer, MMA, second producer
constexpr int kSoftmaxThreads = 256;
constexpr int kProducerWarp = 8, kMmaWarp = 9, kProducer2Warp = 10;
constexpr int kTmemCols = 512;
constexpr int kRingA = 3;      // Q (dK/dV) or K (dQ): used by the first and the last product of a tile
constexpr int kRingB = 2;      // dO (dK/dV) or V (dQ)
constexpr float kLog2e = 1.4426950408889634f;

enum : uint32_t {
    kSiteTcRes = 0x41, kSiteTcAFull = 0x42, kSiteTcAEmpty = 0x43, kSiteTcSFull = 0x44, kSiteTcP = 0x45,
    kSiteTcAcc = 0x46, kSiteTcBFull = 0x47, kSiteTcBEmpty = 0x48, kSiteTcSFree = 0x49, kSiteTcDpFull = 0x4a
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

__device__ __forceinline__ uint32_t dynamic_smem_bytes() {
    uint32_t v;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(v));
    return v;
}

// D = A B^T over K = D columns, both operands K-major 128-row tiles: M = 128, N = 128.
template <int D>
__device__ __forceinline__ void mma_ss_tile(bool leader, uint32_t d_tmem, uint32_t sa, uint32_t sb) {
    constexpr uint32_t idesc = idesc_bf16_f32(kBig, kStep, 0, 0);
    const uint64_t a0 = smem_desc_sw128(sa, 16, 1024), b0 = smem_desc_sw128(sb, 16, 1024);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        // 16 columns = 32 bytes inside a 128-byte row; column groups of 64 are a whole
        // [128 rows][128 B] group apart
        const uint64_t o = (uint64_t)((kk & 3) * 2 + (kk >> 2) * (Tile<D, kBig>::kGroupBytes >> 4));
        mma_bf16_ss(leader, d_tmem, a0 + o, b0 + o, idesc, kk > 0 ? 1u : 0u);
    }
}

// TMEM column of the bf16 pairs for K-block kk (16 rows of the streamed tile) of one
// half, relative to that half's first column: softmax warp group w / 4 = c wrote the
// 32 values of its columns 32 c .. 32 c + 31 as 16 pair columns at 32 c.
__device__ __forceinline__ uint32_t half_col(int kk) { return (uint32_t)((kk >> 1) * 32 + (kk & 1) * 8); }

// D (+)= A B with A = 128 x 64 bf16 in TMEM (half h of the P / dS columns, a_half at
// its first column) and B = rows [64 h, 64 h + 64) of a streamed tile read MN-major
// (K = its rows, N = its D columns).
template <int D>
__device__ __forceinline__ void mma_ts_half(bool leader, uint32_t d_tmem, uint32_t a_half, uint32_t sb, int h,
                                            bool accumulate) {
    constexpr uint32_t idesc = idesc_bf16_f32(kBig, D, 0, 1);
    const uint64_t b0 = smem_desc_sw128(sb, Tile<D, kStep>::kGroupBytes, 1024);
#pragma unroll
    for (int kk = 0; kk < kHalf / 16; ++kk)  // 16 rows of B = 2 KB per step
        mma_bf16_ts(leader, d_tmem, a_half + half_col(kk), b0 + (uint64_t)((h * (kHalf / 16) + kk) * 128), idesc,
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

// dK/dV, step 1 (needs S^T only): P^T = exp2(S^T c - L_col) for one key row over 32
// query columns, in place of the scores (fp32 bits).  l2 points at the 32 columns'
// values in shared memory (the same address in every lane: broadcast loads).
// kMasked: columns col < lim dropped (exponent -inf, weight exactly 0).
template <bool kMasked>
__device__ __forceinline__ void probs_dkdv(uint32_t (&s)[32], const float4* l2, float c, int lim) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float4 L = l2[q];
        const float lv[4] = {L.x, L.y, L.z, L.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int col = 4 * q + e;
            float x = fmaf(__uint_as_float(s[col]), c, -lv[e]);
            if (kMasked) x = col >= lim ? x : -INFINITY;
            s[col] = __float_as_uint(ex2_approx(x));
        }
    }
}

// dK/dV, step 2 (needs dP^T): dS^T = P^T (dP^T - D_col); P^T and dS^T packed to bf16 pairs.
__device__ __forceinline__ void grads_dkdv(const uint32_t (&p)[32], const uint32_t (&dp)[32], const float4* dd,
                                           uint32_t (&pw)[16], uint32_t (&dw)[16]) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float4 Dd = dd[q];
        const float dv[4] = {Dd.x, Dd.y, Dd.z, Dd.w};
        float pf[4], d[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int col = 4 * q + e;
            pf[e] = __uint_as_float(p[col]);
            d[e] = pf[e] * (__uint_as_float(dp[col]) - dv[e]);
        }
        pw[2 * q] = pack_bf16x2(pf[0], pf[1]);
        pw[2 * q + 1] = pack_bf16x2(pf[2], pf[3]);
        dw[2 * q] = pack_bf16x2(d[0], d[1]);
        dw[2 * q + 1] = pack_bf16x2(d[2], d[3]);
    }
}

// dQ, step 1 (needs S only): exp2(S c - L) for one query row over 32 key columns, in
// place of the scores.  kMasked: columns past lim or with a cleared flag byte dropped.
template <bool kMasked>
__device__ __forceinline__ void probs_dq(uint32_t (&s)[32], const uint32_t* keep_w, float c, float l2, int lim) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const uint32_t kw = kMasked ? keep_w[q] : 0xffffffffu;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int col = 4 * q + e;
            float x = fmaf(__uint_as_float(s[col]), c, -l2);
            if (kMasked) x = (col <= lim && ((kw >> (8 * e)) & 0xffu) != 0u) ? x : -INFINITY;
            s[col] = __float_as_uint(ex2_approx(x));
        }
    }
}

// dQ, step 2 (needs dP): dS = P (dP - D) packed to bf16 pairs.
__device__ __forceinline__ void grads_dq(const uint32_t (&p)[32], const uint32_t (&dp)[32], float ddi,
                                         uint32_t (&dw)[16]) {
#pragma unroll
    for (int q = 0; q < 16; ++q)
        dw[q] = pack_bf16x2(__uint_as_float(p[2 * q]) * (__uint_as_float(dp[2 * q]) - ddi),
                            __uint_as_float(p[2 * q + 1]) * (__uint_as_float(dp[2 * q + 1]) - ddi));
}

struct TcBars {
    uint64_t res_full;                      // resident tiles (K, V or Q, dO)
    uint64_t a_full[kRingA], a_empty[kRingA];
    uint64_t b_full[kRingB], b_empty[kRingB];
    uint64_t s_full[2];  // S of a tile computed (dK/dV: one buffer; dQ: two, alternating per tile)
    uint64_t dp_full;    // dP of the current tile computed
    uint64_t s_free[2];  // dK/dV: the softmax warps hold S in registers, so it may be overwritten
                         // ([0] only; dQ's second buffer needs no such handshake)
    uint64_t p_lo, p_hi; // P / dS of a half in TMEM (256 arrivals each)
    uint64_t acc_full;   // last accumulating MMA done
    uint64_t fin;        // abort path: every MMA issued so far done
    uint32_t tmem_base;
    int abort_flag;
};

__device__ __forceinline__ void init_bars(TcBars& bar) {
    mbar_init(&bar.res_full, 1);
    for (int s = 0; s < kRingA; ++s) {
        mbar_init(&bar.a_full[s], 1);
        mbar_init(&bar.a_empty[s], 1);
    }
    for (int s = 0; s < kRingB; ++s) {
        mbar_init(&bar.b_full[s], 1);
        mbar_init(&bar.b_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
        mbar_init(&bar.s_full[s], 1);
        mbar_init(&bar.s_free[s], kSoftmaxThreads);
    }
    mbar_init(&bar.dp_full, 1);
    mbar_init(&bar.p_lo, kSoftmaxThreads);
    mbar_init(&bar.p_hi, kSoftmaxThreads);
    mbar_init(&bar.acc_full, 1);
    mbar_init(&bar.fin, 1);
    bar.abort_flag = 0;
    fence_mbar_init();
}

// On an abort, let the copies a producer has in flight land before the CTA exits.
__device__ __forceinline__ void drain_ring(uint64_t* full, int ring, int issued) {
    for (int t = max(0, issued - ring); t < issued; ++t) mbar_drain(&full[t % ring], (t / ring) & 1);
}

template <int D>
struct DkdvTcSmem {
    static constexpr int kBigT = Tile<D, kBig>::kBytes, kStepT = Tile<D, kStep>::kBytes;
    static constexpr int kOffK = 0, kOffV = kBigT, kOffQ = 2 * kBigT, kOffO = kOffQ + kRingA * kStepT;
    static constexpr int kOffL2 = kOffO + kRingB * kStepT;        // float l2[kRingA][128], with the Q stages
    static constexpr int kOffDD = kOffL2 + kRingA * kStep * 4;     // float dd[kRingB][128], with the dO stages
    static constexpr int kOffBar = kOffDD + kRingB * kStep * 4;
    static constexpr int kBytes = kOffBar + (int)sizeof(TcBars);
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo, const BwdArgs a,
                unsigned int* status) {
    using L = DkdvTcSmem<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    // at d = 128 the layout leaves less than 1 KB of the largest allocation for the
    // 1024-byte alignment the swizzled tiles need: refuse (uniformly, before any
    // barrier, copy or TMEM allocation) if this launch's base does not allow it
    if (pad + (uint32_t)L::kBytes > dynamic_smem_bytes()) {
        if (threadIdx.x == 0) atomicOr(status, ATTN_DEV_SMEM_LAYOUT);
        return;
    }
    uint8_t* smem = smem_raw + pad;
    float* s_l2 = reinterpret_cast<float*>(smem + L::kOffL2);   // [kRingA][128]
    float* s_dd = reinterpret_cast<float*>(smem + L::kOffDD);   // [kRingB][128]
    TcBars& bar = *reinterpret_cast<TcBars*>(smem + L::kOffBar);
    volatile int* ab = &bar.abort_flag;

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int n_kb = (a.n_kv + kBig - 1) / kBig;
    const int per = a.H_kv * a.B;
    const int kb = blockIdx.x / per;   // the first key blocks are the heaviest under a causal mask: first
    const int g = (blockIdx.x % per) % a.H_kv, b = (blockIdx.x % per) / a.H_kv;
    if (kb >= n_kb) return;
    // the dQ kernel does not read this kernel's results: it may fill SMs this grid's last
    // blocks leave idle
    grid_dependents_launch();
    const int j0 = kb * kBig;
    const int group = a.H / a.H_kv;
    const int off = a.n_kv - a.n_q;    // causal: key j is visible to query i when j <= i + off
    const int n_qb = (a.n_q + kStep - 1) / kStep;
    const int qb0 = a.causal ? max(0, j0 - off) / kStep : 0;
    const int per_head = n_qb - qb0;
    const int steps = group * per_head;   // >= 1: row n_q - 1 sees every key when causal
    // query tile t of the CTA: the group's heads one after another, each from its first
    // visible query tile to its last
    auto tile_head = [&](int t) { return g * group + t / per_head; };
    auto tile_qb = [&](int t) { return qb0 + t % per_head; };
    // workspace row of the first query of tile t
    auto ws_row = [&](int t) {
        return ((size_t)b * a.H + (size_t)tile_head(t)) * a.n_q_pad + (size_t)tile_qb(t) * kStep;
    };

    if (tid == 0) init_bars(bar);
    if (warp == kMmaWarp) {
        tmem_alloc(&bar.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar.tmem_base;
    constexpr uint32_t kColDV = 0, kColDK = D, kColS = 2 * D, kColP = 2 * D + kStep;   // dP^T, then P^T / dS^T

    if (warp == kProducerWarp) {
        if (lane == 0) {
            int issued = 0;
            bool ok = true;
            mbar_arrive_expect_tx(&bar.res_full, 2 * L::kBigT);
            tma_tile<D, kBig>(smem + L::kOffK, &tk, &bar.res_full, j0, g, b);
            tma_tile<D, kBig>(smem + L::kOffV, &tv, &bar.res_full, j0, g, b);
            for (int t = 0; t < steps; ++t) {
                const int st = t % kRingA;
                if (!mbar_wait(&bar.a_empty[st], ((t / kRingA) & 1) ^ 1, ab, status, kSiteTcAEmpty)) {
                    ok = false;
                    break;
                }
                const int h = tile_head(t), qb = tile_qb(t);
                mbar_arrive_expect_tx(&bar.a_full[st], L::kStepT + kStep * 4);
                tma_tile<D, kStep>(smem + L::kOffQ + st * L::kStepT, &tq, &bar.a_full[st], qb * kStep, h, b);
                bulk_load(s_l2 + st * kStep, a.ws_l2 + ws_row(t), kStep * 4, &bar.a_full[st]);
                issued = t + 1;
            }
            if (!ok || *ab) {
                mbar_drain(&bar.res_full, 0);
                drain_ring(bar.a_full, kRingA, issued);
            }
        }
    } else if (warp == kProducer2Warp) {
        if (lane == 0) {
            int issued = 0;
            bool ok = true;
            for (int t = 0; t < steps; ++t) {
                const int st = t % kRingB;
                if (!mbar_wait(&bar.b_empty[st], ((t / kRingB) & 1) ^ 1, ab, status, kSiteTcBEmpty)) {
                    ok = false;
                    break;
                }
                const int h = tile_head(t), qb = tile_qb(t);
                mbar_arrive_expect_tx(&bar.b_full[st], L::kStepT + kStep * 4);
                tma_tile<D, kStep>(smem + L::kOffO + st * L::kStepT, &tdo, &bar.b_full[st], qb * kStep, h, b);
                bulk_load(s_dd + st * kStep, a.ws_dd + ws_row(t), kStep * 4, &bar.b_full[st]);
                issued = t + 1;
            }
            if (!ok || *ab) drain_ring(bar.b_full, kRingB, issued);
        }
    } else if (warp == kMmaWarp) {
        const bool leader = lane == 0;
        const uint32_t sK = smem_u32(smem + L::kOffK), sV = smem_u32(smem + L::kOffV);
        auto sQ = [&](int t) { return smem_u32(smem + L::kOffQ + (t % kRingA) * L::kStepT); };
        auto sO = [&](int t) { return smem_u32(smem + L::kOffO + (t % kRingB) * L::kStepT); };
        bool ok = warp_wait(&bar.res_full, 0, ab, status, kSiteTcRes) &&
                  warp_wait(&bar.a_full[0], 0, ab, status, kSiteTcAFull);
        if (ok) {
            tc_fence_after();
            mma_ss_tile<D>(leader, tmem + kColS, sK, sQ(0));   // S^T = K Q^T
            mma_commit(leader, &bar.s_full[0]);
            ok = warp_wait(&bar.b_full[0], 0, ab, status, kSiteTcBFull);
        }
        if (ok) {
            tc_fence_after();
            mma_ss_tile<D>(leader, tmem + kColP, sV, sO(0));   // dP^T = V dO^T
            mma_commit(leader, &bar.dp_full);
        }
        for (int t = 0; ok && t < steps; ++t) {
            const uint32_t ph = (uint32_t)t & 1u;
            if (t + 1 < steps) {
                ok = warp_wait(&bar.a_full[(t + 1) % kRingA], ((t + 1) / kRingA) & 1, ab, status, kSiteTcAFull) &&
                     warp_wait(&bar.s_free[0], ph, ab, status, kSiteTcSFree);
                if (!ok) break;
                tc_fence_after();
                mma_ss_tile<D>(leader, tmem + kColS, sK, sQ(t + 1));
                mma_commit(leader, &bar.s_full[0]);
            }
            ok = warp_wait(&bar.p_lo, ph, ab, status, kSiteTcP);
            if (!ok) break;
            tc_fence_after();
            mma_ts_half<D>(leader, tmem + kColDV, tmem + kColP, sO(t), 0, t > 0);        // dV += P^T dO
            mma_ts_half<D>(leader, tmem + kColDK, tmem + kColP + 16, sQ(t), 0, t > 0);   // dK += dS^T Q
            ok = warp_wait(&bar.p_hi, ph, ab, status, kSiteTcP);
            if (!ok) break;
            tc_fence_after();
            mma_ts_half<D>(leader, tmem + kColDV, tmem + kColP + kHalf, sO(t), 1, true);
            mma_ts_half<D>(leader, tmem + kColDK, tmem + kColP + kHalf + 16, sQ(t), 1, true);
            mma_commit(leader, &bar.a_empty[t % kRingA]);
            mma_commit(leader, &bar.b_empty[t % kRingB]);
            if (t == steps - 1) mma_commit(leader, &bar.acc_full);
            if (t + 1 < steps) {
                ok = warp_wait(&bar.b_full[(t + 1) % kRingB], ((t + 1) / kRingB) & 1, ab, status, kSiteTcBFull);
                if (!ok) break;
                tc_fence_after();
                mma_ss_tile<D>(leader, tmem + kColP, sV, sO(t + 1));   // after the products that read P / dS
                mma_commit(leader, &bar.dp_full);
            }
        }
        if (!ok) {
            mma_commit(leader, &bar.fin);
            if (leader) mbar_drain(&bar.fin, 0);
        }
        __syncwarp();
    } else {
        // softmax warps: thread = key row j0 + 32 (warp % 4) + lane (TMEM lane 32 (warp % 4) + lane);
        // columns 32 c .. 32 c + 31 of each half, c = warp / 4
        const int quarter = warp % 4, c = warp / 4;
        const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
        const int j = j0 + 32 * quarter + lane;
        const bool key_ok = j < a.n_kv && (a.key_mask == nullptr || a.key_mask[(size_t)b * a.n_kv + j] != 0);
        const float cs = a.scale * kLog2e;
        bool ok = true;
        for (int t = 0; t < steps; ++t) {
            const uint32_t ph = (uint32_t)t & 1u;
            ok = mbar_wait(&bar.s_full[0], ph, ab, status, kSiteTcSFull);
            if (!__all_sync(0xffffffffu, ok)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t p_lo[32], p_hi[32];
            tmem_ld32(tmem + lane_off + kColS + 32 * c, p_lo);
            tmem_ld32(tmem + lane_off + kColS + kHalf + 32 * c, p_hi);
            tmem_wait_ld();
            pin(p_lo);
            pin(p_hi);
            tc_fence_before();
            mbar_arrive(&bar.s_free[0]);
            // a_full of this tile (already complete: S used its stage) makes the stage's
            // l2 row visible to this thread
            ok = mbar_wait(&bar.a_full[t % kRingA], (t / kRingA) & 1, ab, status, kSiteTcAFull);
            if (!__all_sync(0xffffffffu, ok)) {
                ok = false;
                break;
            }
            const int i0 = tile_qb(t) * kStep;
            const bool diag = a.causal && (j0 + kBig - 1 - off > i0);
            // query column col is kept iff col >= lim (a masked key row keeps none)
            const int lim = !key_ok ? kStep : (diag ? j - off - i0 : 0);
            const float4* l2_t = reinterpret_cast<const float4*>(s_l2 + (t % kRingA) * kStep);
            // the exponentials run while the tensor core computes dP^T
            if (__all_sync(0xffffffffu, lim <= 32 * c)) {
                probs_dkdv<false>(p_lo, l2_t + 8 * c, cs, 0);
            } else {
                probs_dkdv<true>(p_lo, l2_t + 8 * c, cs, lim - 32 * c);
            }
            if (__all_sync(0xffffffffu, lim <= kHalf + 32 * c)) {
                probs_dkdv<false>(p_hi, l2_t + 16 + 8 * c, cs, 0);
            } else {
                probs_dkdv<true>(p_hi, l2_t + 16 + 8 * c, cs, lim - kHalf - 32 * c);
            }
            ok = mbar_wait(&bar.dp_full, ph, ab, status, kSiteTcDpFull) &&
                 mbar_wait(&bar.b_full[t % kRingB], (t / kRingB) & 1, ab, status, kSiteTcBFull);
            if (!__all_sync(0xffffffffu, ok)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const float4* dd_t = reinterpret_cast<const float4*>(s_dd + (t % kRingB) * kStep);
            auto half = [&](const uint32_t (&pv)[32], int col0, uint64_t* ready) {
                uint32_t dp[32], pw[16], dw[16];
                tmem_ld32(tmem + lane_off + kColP + col0, dp);
                tmem_wait_ld();
                pin(dp);
                grads_dkdv(pv, dp, dd_t + col0 / 4, pw, dw);
                // over this warp's own dP^T columns, already in registers
                tmem_st16(tmem + lane_off + kColP + col0, pw);
                tmem_st16(tmem + lane_off + kColP + col0 + 16, dw);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(ready);
            };
            half(p_lo, 32 * c, &bar.p_lo);
            half(p_hi, kHalf + 32 * c, &bar.p_hi);
        }
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bar.acc_full, 0, ab, status, kSiteTcAcc));
        if (ok) {
            tc_fence_after();
            __nv_bfloat16* dk_row = static_cast<__nv_bfloat16*>(a.dk) + (((size_t)b * a.H_kv + g) * a.n_kv + j) * D;
            __nv_bfloat16* dv_row = static_cast<__nv_bfloat16*>(a.dv) + (((size_t)b * a.H_kv + g) * a.n_kv + j) * D;
#pragma unroll
            for (int c0 = c * (D / 2); c0 < (c + 1) * (D / 2); c0 += 32) {
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
    static constexpr int kOffQ = 0, kOffO = kBigT, kOffK = 2 * kBigT, kOffV = kOffK + kRingA * kStepT;
    static constexpr int kOffKeep = kOffV + kRingB * kStepT;   // uint8 keep[kRingA][128]
    static constexpr int kOffBar = kOffKeep + kRingA * kStep;
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
    uint8_t* s_keep = smem + L::kOffKeep;   // [kRingA][128]
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

    if (tid == 0) init_bars(bar);
    if (warp == kMmaWarp) {
        tmem_alloc(&bar.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar.tmem_base;
    // S is double-buffered (two tiles' scores), so the next S never waits for the softmax
    // warps to pick up the current one
    constexpr uint32_t kColDQ = 0, kColP = D + 2 * kStep;   // dP, then dS
    auto colS = [](int t) { return (uint32_t)(D + (t & 1) * kStep); };

    if (warp == kProducerWarp) {
        int issued = 0;
        bool ok = true;
        if (lane == 0 && n_kb > 0) {
            mbar_arrive_expect_tx(&bar.res_full, 2 * L::kBigT);
            tma_tile<D, kBig>(smem + L::kOffQ, &tq, &bar.res_full, q0, h, b);
            tma_tile<D, kBig>(smem + L::kOffO, &tdo, &bar.res_full, q0, h, b);
        }
        for (int t = 0; t < n_kb; ++t) {
            const int st = t % kRingA;
            ok = warp_wait(&bar.a_empty[st], ((t / kRingA) & 1) ^ 1, ab, status, kSiteTcAEmpty);
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
                mbar_arrive_expect_tx(&bar.a_full[st], L::kStepT);
                tma_tile<D, kStep>(smem + L::kOffK + st * L::kStepT, &tk, &bar.a_full[st], t * kStep, g, b);
            }
            issued = t + 1;
        }
        if (lane == 0 && (!ok || *ab)) {
            if (n_kb > 0) mbar_drain(&bar.res_full, 0);
            drain_ring(bar.a_full, kRingA, issued);
        }
    } else if (warp == kProducer2Warp) {
        if (lane == 0) {
            int issued = 0;
            bool ok = true;
            for (int t = 0; t < n_kb; ++t) {
                const int st = t % kRingB;
                if (!mbar_wait(&bar.b_empty[st], ((t / kRingB) & 1) ^ 1, ab, status, kSiteTcBEmpty)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&bar.b_full[st], L::kStepT);
                tma_tile<D, kStep>(smem + L::kOffV + st * L::kStepT, &tv, &bar.b_full[st], t * kStep, g, b);
                issued = t + 1;
            }
            if (!ok || *ab) drain_ring(bar.b_full, kRingB, issued);
        }
    } else if (warp == kMmaWarp) {
        const bool leader = lane == 0;
        const uint32_t sQ = smem_u32(smem + L::kOffQ), sO = smem_u32(smem + L::kOffO);
        auto sK = [&](int t) { return smem_u32(smem + L::kOffK + (t % kRingA) * L::kStepT); };
        auto sV = [&](int t) { return smem_u32(smem + L::kOffV + (t % kRingB) * L::kStepT); };
        bool ok = true;
        if (n_kb > 0) {
            ok = warp_wait(&bar.res_full, 0, ab, status, kSiteTcRes) &&
                 warp_wait(&bar.a_full[0], 0, ab, status, kSiteTcAFull);
            if (ok) {
                tc_fence_after();
                mma_ss_tile<D>(leader, tmem + colS(0), sQ, sK(0));   // S = Q K^T
                mma_commit(leader, &bar.s_full[0]);
                ok = warp_wait(&bar.b_full[0], 0, ab, status, kSiteTcBFull);
            }
            if (ok) {
                tc_fence_after();
                mma_ss_tile<D>(leader, tmem + kColP, sO, sV(0));   // dP = dO V^T
                mma_commit(leader, &bar.dp_full);
                mma_commit(leader, &bar.b_empty[0]);               // V is read by dP alone
            }
        }
        for (int t = 0; ok && t < n_kb; ++t) {
            const uint32_t ph = (uint32_t)t & 1u;
            if (t + 1 < n_kb) {
                // S_{t+1} goes into the buffer S_{t-1} used.  Every softmax thread loaded S_{t-1}
                // (tcgen05.wait::ld, fence) before it arrived on p_hi for tile t - 1, which this
                // warp waited for in the previous iteration: the buffer is free.
                const int u = t + 1;
                ok = warp_wait(&bar.a_full[u % kRingA], (u / kRingA) & 1, ab, status, kSiteTcAFull);
                if (!ok) break;
                tc_fence_after();
                mma_ss_tile<D>(leader, tmem + colS(u), sQ, sK(u));
                mma_commit(leader, &bar.s_full[u & 1]);
            }
            ok = warp_wait(&bar.p_lo, ph, ab, status, kSiteTcP);
            if (!ok) break;
            tc_fence_after();
            mma_ts_half<D>(leader, tmem + kColDQ, tmem + kColP, sK(t), 0, t > 0);   // dQ += dS K
            ok = warp_wait(&bar.p_hi, ph, ab, status, kSiteTcP);
            if (!ok) break;
            tc_fence_after();
            mma_ts_half<D>(leader, tmem + kColDQ, tmem + kColP + kHalf, sK(t), 1, true);
            mma_commit(leader, &bar.a_empty[t % kRingA]);
            if (t == n_kb - 1) mma_commit(leader, &bar.acc_full);
            if (t + 1 < n_kb) {
                ok = warp_wait(&bar.b_full[(t + 1) % kRingB], ((t + 1) / kRingB) & 1, ab, status, kSiteTcBFull);
                if (!ok) break;
                tc_fence_after();
                mma_ss_tile<D>(leader, tmem + kColP, sO, sV(t + 1));   // after the products that read dS
                mma_commit(leader, &bar.dp_full);
                mma_commit(leader, &bar.b_empty[(t + 1) % kRingB]);
            }
        }
        if (!ok) {
            mma_commit(leader, &bar.fin);
            if (leader) mbar_drain(&bar.fin, 0);
        }
        __syncwarp();
    } else {
        // softmax warps: thread = query row q0 + 32 (warp % 4) + lane; columns 32 c .. 32 c + 31
        // of each half, c = warp / 4
        const int quarter = warp % 4, c = warp / 4;
        const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
        const int i = q0 + 32 * quarter + lane;
        const size_t lrow = ((size_t)b * a.H + h) * a.n_q_pad + i;
        const bool row_in = i < a.n_q;
        const float l2 = row_in ? a.ws_l2[lrow] : INFINITY;   // rows past n_q: weight 0
        const float ddi = row_in ? a.ws_dd[lrow] : 0.f;
        const float cs = a.scale * kLog2e;
        bool ok = true;
        for (int t = 0; t < n_kb; ++t) {
            const uint32_t ph = (uint32_t)t & 1u;
            const int st = t % kRingA;
            ok = mbar_wait(&bar.s_full[t & 1], (t >> 1) & 1, ab, status, kSiteTcSFull);
            if (!__all_sync(0xffffffffu, ok)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t p_lo[32], p_hi[32];
            tmem_ld32(tmem + lane_off + colS(t) + 32 * c, p_lo);
            tmem_ld32(tmem + lane_off + colS(t) + kHalf + 32 * c, p_hi);
            tmem_wait_ld();
            pin(p_lo);
            pin(p_hi);
            // a_full[st] (already complete: S used the stage) makes the key flags visible
            ok = mbar_wait(&bar.a_full[st], (t / kRingA) & 1, ab, status, kSiteTcAFull);
            if (!__all_sync(0xffffffffu, ok)) {
                ok = false;
                break;
            }
            const int j0 = t * kStep;
            const bool diag = a.causal && (j0 + kStep - 1 > q0 + off);
            // key column col is kept iff col <= lim and its flag is set (a key mask or the
            // end of the keys clears flags); dropped entries get exponent -inf, weight 0
            const int lim = diag ? i + off - j0 : kStep;
            const bool flags_all = (a.key_mask == nullptr) && (j0 + kStep <= a.n_kv);
            const uint32_t* keep_w = reinterpret_cast<const uint32_t*>(s_keep + st * kStep);
            // the exponentials run while the tensor core computes dP
            if (flags_all && __all_sync(0xffffffffu, lim >= 32 * c + 31))
                probs_dq<false>(p_lo, keep_w + 8 * c, cs, l2, 31);
            else
                probs_dq<true>(p_lo, keep_w + 8 * c, cs, l2, lim - 32 * c);
            if (flags_all && __all_sync(0xffffffffu, lim >= kHalf + 32 * c + 31))
                probs_dq<false>(p_hi, keep_w + 16 + 8 * c, cs, l2, 31);
            else
                probs_dq<true>(p_hi, keep_w + 16 + 8 * c, cs, l2, lim - kHalf - 32 * c);
            ok = mbar_wait(&bar.dp_full, ph, ab, status, kSiteTcDpFull);
            if (!__all_sync(0xffffffffu, ok)) {
                ok = false;
                break;
            }
            tc_fence_after();
            auto half = [&](const uint32_t (&pv)[32], int col0, uint64_t* ready) {
                uint32_t dp[32], dw[16];
                tmem_ld32(tmem + lane_off + kColP + col0, dp);
                tmem_wait_ld();
                pin(dp);
                grads_dq(pv, dp, ddi, dw);
                tmem_st16(tmem + lane_off + kColP + col0, dw);   // over this warp's own dP columns
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(ready);
            };
            half(p_lo, 32 * c, &bar.p_lo);
            half(p_hi, kHalf + 32 * c, &bar.p_hi);
        }
        if (ok && n_kb > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bar.acc_full, 0, ab, status, kSiteTcAcc));
        if (ok) {
            __nv_bfloat16* dq_row = static_cast<__nv_bfloat16*>(a.dq) + (((size_t)b * a.H + h) * a.n_q + i) * D;
            if (n_kb == 0) {
                if (row_in) {
                    uint4* d4 = reinterpret_cast<uint4*>(dq_row + c * (D / 2));
                    for (int k = 0; k < D / 16; ++k) d4[k] = make_uint4(0u, 0u, 0u, 0u);
                }
            } else {
                tc_fence_after();
#pragma unroll
                for (int c0 = c * (D / 2); c0 < (c + 1) * (D / 2); c0 += 32) {
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
    // launched as a programmatic dependent of the dK/dV kernel, which it does not read: it
    // finishes only after that grid, so work queued after the backward sees both
    grid_dependency_wait();
}

template <int D>
cudaError_t launch_tc_d(const BwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                        const CUtensorMap& tdo, unsigned int* status, cudaStream_t stream) {
    // more than half of an SM's shared memory: one CTA per SM, so the 512-column
    // TMEM allocation never waits for another CTA
    static std::atomic<unsigned long long> ready{0};
    static std::atomic<int> optin_smem[64];
    const int smem_q = std::max(DqTcSmem<D>::kBytes + 1024, 118 * 1024);
    auto kv_bytes = [](int optin) { return std::min(std::max(DkdvTcSmem<D>::kBytes + 1024, 118 * 1024), optin); };
    int dev = 0;
    cudaError_t e = setup_once_per_device(ready, &dev, [smem_q, kv_bytes](int device) {
        int optin = 0;
        cudaError_t r = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
        if (r == cudaSuccess)
            r = cudaFuncSetAttribute(bwd_dkdv_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, kv_bytes(optin));
        if (r == cudaSuccess) r = cudaFuncSetAttribute(bwd_dq_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_q);
        if (r == cudaSuccess && device < 64) optin_smem[device].store(optin, std::memory_order_relaxed);
        return r;
    });
    if (e != cudaSuccess) return e;
    int optin = dev < 64 ? optin_smem[dev].load(std::memory_order_relaxed) : 0;
    if (optin <= 0) {
        e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess) return e;
    }
    const int smem_kv = kv_bytes(optin);
    const long long grid_kv = (long long)((a.n_kv + kBig - 1) / kBig) * a.H_kv * a.B;
    const long long grid_q = (long long)((a.n_q + kBig - 1) / kBig) * a.H * a.B;
    if (grid_kv > 0x7fffffffll || grid_q > 0x7fffffffll) return cudaErrorInvalidConfiguration;
    bwd_dkdv_tc<D><<<(unsigned)grid_kv, kThreads, smem_kv, stream>>>(tq, tk, tv, tdo, a, status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid_q, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem_q;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, bwd_dq_tc<D>, tq, tk, tv, tdo, a, status);
    if (e != cudaSuccess) return e;
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
