// bf16 forward attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Method: the blocked online softmax ("Sviluppo AI ed Algebra Lineare",
// sections "Tiling" and "Online Softmax (La Formalizzazione Matematica)"; the
// (m, l, u) invariant of "Attenzione: softmax online, riscalamento e memoria",
// section 2).  For a 128-row query tile the kernel walks the key/value blocks;
// for each block it forms S = Q K^T, updates the running row maximum m and
// normaliser l, rescales the unnormalised output u (held in TMEM) by
// 2^(m_old - m_new) whenever the maximum grows, and adds P V with
// P = 2^(S * scale * log2(e) - m).  Normalisation by l happens once at the end
// (deferred normalisation, "Sviluppo AI ed Algebra Lineare", FlashAttention-2
// section), as does the log-sum-exp.
//
// B200 mapping (one CTA per 128-row query tile, 6 warps):
//   warp 4       TMA producer: Q once, then K_j and V_j through a 2-stage
//                shared-memory ring (128-byte swizzle, mbarrier expect_tx)
//   warp 5       TMEM allocator and single-thread tcgen05.mma issuer:
//                S_j = Q K_j^T (both operands K-major in shared memory) into one
//                of two TMEM score buffers, then O += P_{j-1} V_{j-1} with P read
//                from TMEM and V MN-major in shared memory
//   warps 0-3    softmax / correction / epilogue: thread t owns query row t
//                (TMEM lane t); loads its score row, masks, takes the row
//                maximum, writes P (bf16) over the first half of the same TMEM
//                buffer, rescales its O row when needed and finally writes
//                O / l (bf16) and the log-sum-exp.
// The tensor core computes S_{j+1} while the softmax warps work on S_j.
#include <algorithm>
#include <cmath>
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace attn {
namespace {

using namespace dev;

constexpr int BM = 128;          // query rows per tile (= TMEM lanes)
constexpr int BN = 128;          // keys per block
constexpr int kStages = 2;       // K/V ring depth
constexpr int kThreads = 192;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
constexpr int kSubBytes = 128 * 128;  // one [128 rows][64 bf16] swizzled sub-tile = 16 KB
constexpr float kLog2e = 1.4426950408889634f;

// Codes of the wait sites, recorded if a bounded wait gives up.
enum WaitSite : uint32_t {
    kSiteKEmpty = 1, kSiteVEmpty, kSiteQFull, kSiteKFull, kSitePFull, kSiteVFull, kSiteSFull, kSiteOFull,
    kSiteOFinal
};
// Debug progress slots (written by block 0 only, when a trace buffer is set).
enum TraceSlot : int {
    kTrInit = 0, kTrAlloc, kTrBlocks, kTrProducer, kTrMma, kTrSoftmax, kTrEpilogue, kTrExit
};

template <int D>
struct Layout {
    static constexpr int kSubs = D / 64;                  // 64-column sub-tiles per row block
    static constexpr int kTileBytes = kSubs * kSubBytes;  // a [128][D] bf16 tile
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kTileBytes;
    static constexpr int kOffV = kOffK + kStages * kTileBytes;
    static constexpr int kOffBar = kOffV + kStages * kTileBytes;
    static constexpr int kBytes = kOffBar + 256;
};

struct Bars {
    uint64_t q_full;
    uint64_t k_full[kStages], k_empty[kStages];
    uint64_t v_full[kStages], v_empty[kStages];
    uint64_t s_full[2], p_full[2];
    uint64_t o_full;
    uint32_t tmem_base;
    int abort_flag;
    int first_unkept;   // smallest masked-out key index (n_kv if none)
    int last_kept;      // largest kept key index (-1 if none)
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_bf16_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                    const __grid_constant__ CUtensorMap tv, const FwdArgs a, unsigned int* status) {
    using L = Layout<D>;
    extern __shared__ uint8_t smem_raw[];
    // tiles need 1024-byte alignment for the 128-byte swizzle atoms
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    Bars& bar = *reinterpret_cast<Bars*>(smem + L::kOffBar);

    const int tid = threadIdx.x;
    const int warp = tid / 32;
    const int n_mblk = (a.n_q + BM - 1) / BM;
    const int mblk = a.causal ? (n_mblk - 1 - (int)blockIdx.x) : (int)blockIdx.x;  // heavy causal tiles first
    const int h = blockIdx.y, b = blockIdx.z;
    const int g = h / (a.H / a.H_kv);
    const int m0 = mblk * BM;
    const int offset = a.n_kv - a.n_q;  // causal: row i sees keys j <= i + offset

    if (tid == 0) {
        mbar_init(&bar.q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bar.k_full[s], 1);
            mbar_init(&bar.k_empty[s], 1);
            mbar_init(&bar.v_full[s], 1);
            mbar_init(&bar.v_empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar.s_full[i], 1);
            mbar_init(&bar.p_full[i], 128);
        }
        mbar_init(&bar.o_full, 1);
        bar.abort_flag = 0;
        bar.first_unkept = a.n_kv;
        bar.last_kept = a.key_mask ? -1 : a.n_kv - 1;
        fence_mbar_init();
    }
    unsigned int* const trace = (blockIdx.x | blockIdx.y | blockIdx.z) == 0 ? a.trace : nullptr;
    if (tid == 0) trace_mark(trace, kTrInit, 1);
    if (warp == kMmaWarp) {
        tmem_alloc(&bar.tmem_base, kTmemCols);
        tmem_relinquish();
        if (tid % 32 == 0) trace_mark(trace, kTrAlloc, 1);
    }
    __syncthreads();
    if (a.key_mask != nullptr) {
        // summarise this batch row's key mask: first excluded and last kept key
        const uint8_t* km = a.key_mask + (size_t)b * a.n_kv;
        int fu = a.n_kv, lk = -1;
        for (int j = tid; j < a.n_kv; j += kThreads) {
            if (km[j]) lk = j;
            else if (fu == a.n_kv) fu = j;
        }
        if (fu < a.n_kv) atomicMin(&bar.first_unkept, fu);
        if (lk >= 0) atomicMax(&bar.last_kept, lk);
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar.tmem_base;

    // key blocks this tile visits
    int kv_hi = min(a.n_kv, bar.last_kept + 1);
    if (a.causal) kv_hi = min(kv_hi, m0 + BM + offset);
    const int n_blk = kv_hi > 0 ? (kv_hi + BN - 1) / BN : 0;
    const int first_unkept = bar.first_unkept;
    if (tid == 0) trace_mark(trace, kTrBlocks, 0x10000u | (uint32_t)n_blk);

    const uint32_t sQ = smem_u32(smem + L::kOffQ);
    const uint32_t sK = smem_u32(smem + L::kOffK);
    const uint32_t sV = smem_u32(smem + L::kOffV);

    if (warp == kProducerWarp) {
        if (tid % 32 == 0 && n_blk > 0) {
            tma_prefetch_desc(&tq);
            tma_prefetch_desc(&tk);
            tma_prefetch_desc(&tv);
            mbar_arrive_expect_tx(&bar.q_full, L::kTileBytes);
#pragma unroll
            for (int s = 0; s < L::kSubs; ++s)
                tma_load_4d(smem + L::kOffQ + s * kSubBytes, &tq, &bar.q_full, s * 64, m0, h, b);
            int issued_k = 0, issued_v = 0;  // blocks whose K / V loads were issued
            for (int j = 0; j < n_blk; ++j) {
                const int st = j % kStages;
                const uint32_t ph = (j / kStages) & 1;
                if (!mbar_wait(&bar.k_empty[st], ph ^ 1, &bar.abort_flag, status, kSiteKEmpty)) break;
                mbar_arrive_expect_tx(&bar.k_full[st], L::kTileBytes);
#pragma unroll
                for (int s = 0; s < L::kSubs; ++s)
                    tma_load_4d(smem + L::kOffK + st * L::kTileBytes + s * kSubBytes, &tk, &bar.k_full[st], s * 64,
                                j * BN, g, b);
                issued_k = j + 1;
                if (!mbar_wait(&bar.v_empty[st], ph ^ 1, &bar.abort_flag, status, kSiteVEmpty)) break;
                mbar_arrive_expect_tx(&bar.v_full[st], L::kTileBytes);
#pragma unroll
                for (int s = 0; s < L::kSubs; ++s)
                    tma_load_4d(smem + L::kOffV + st * L::kTileBytes + s * kSubBytes, &tv, &bar.v_full[st], s * 64,
                                j * BN, g, b);
                issued_v = j + 1;
                trace_mark(trace, kTrProducer, (uint32_t)issued_v);
            }
            if (bar.abort_flag) {
                // an aborted CTA must not exit with its bulk copies still landing in shared memory
                mbar_drain(&bar.q_full, 0);
                for (int j = max(0, issued_k - kStages); j < issued_k; ++j)
                    mbar_drain(&bar.k_full[j % kStages], (j / kStages) & 1);
                for (int j = max(0, issued_v - kStages); j < issued_v; ++j)
                    mbar_drain(&bar.v_full[j % kStages], (j / kStages) & 1);
            }
        }
    } else if (warp == kMmaWarp) {
        if (tid % 32 == 0 && n_blk > 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(BM, BN, 0, 0);
            constexpr uint32_t idesc_o = idesc_bf16_f32(BM, D, 0, 1);
            bool ok = mbar_wait(&bar.q_full, 0, &bar.abort_flag, status, kSiteQFull);
            for (int j = 0; ok && j <= n_blk; ++j) {
                if (j < n_blk) {
                    const int st = j % kStages;
                    const int buf = j & 1;
                    if (!mbar_wait(&bar.k_full[st], (j / kStages) & 1, &bar.abort_flag, status, kSiteKFull)) break;
                    tc_fence_after();
                    const uint32_t kbase = sK + st * L::kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t koff = (kk / 4) * kSubBytes + (kk % 4) * 32;
                        const uint64_t ad = smem_desc_sw128(sQ + koff, 16, 1024);
                        const uint64_t bd = smem_desc_sw128(kbase + koff, 16, 1024);
                        mma_bf16_ss(tmem + (buf ? kColS1 : kColS0), ad, bd, idesc_s, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&bar.s_full[buf]);
                    mma_commit(&bar.k_empty[st]);
                    trace_mark(trace, kTrMma, 2u * j + 1u);
                }
                if (j >= 1) {
                    const int jp = j - 1;
                    const int st = jp % kStages;
                    const int buf = jp & 1;
                    if (!mbar_wait(&bar.p_full[buf], (jp >> 1) & 1, &bar.abort_flag, status, kSitePFull)) break;
                    if (!mbar_wait(&bar.v_full[st], (jp / kStages) & 1, &bar.abort_flag, status, kSiteVFull)) break;
                    tc_fence_after();
                    const uint32_t vbase = sV + st * L::kTileBytes;
                    const uint32_t pcol = buf ? kColS1 : kColS0;
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk) {
                        // 16 keys per step: 8 packed bf16x2 TMEM columns of P, 16 rows of V
                        const uint64_t bd = smem_desc_sw128(vbase + kk * 16 * 128, kSubBytes, 1024);
                        mma_bf16_ts(tmem + kColO, tmem + pcol + kk * 8, bd, idesc_o, (jp > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(&bar.v_empty[st]);
                    mma_commit(&bar.o_full);
                    trace_mark(trace, kTrMma, 2u * jp + 2u);
                }
            }
        }
    } else {
        // ------------------------------------------------ softmax warpgroup (warps 0-3)
        const int r = tid;                 // row within the tile = TMEM lane
        const int row = m0 + r;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const float sl2 = a.scale * kLog2e;
        const int row_limit = a.causal ? row + offset : 0x7fffffff;
        float m_run = -INFINITY;  // running maximum, base-2 units of the scaled score
        float l_run = 0.f;
        bool ok = true;

        for (int j = 0; j < n_blk; ++j) {
            const int buf = j & 1;
            const uint32_t scol = buf ? kColS1 : kColS0;
            if (!warp_wait(&bar.s_full[buf], (j >> 1) & 1, &bar.abort_flag, status, kSiteSFull)) { ok = false; break; }
            tc_fence_after();
            uint32_t sraw[BN];
            tmem_ld32(tmem + lane_base + scol + 0, sraw + 0);
            tmem_ld32(tmem + lane_base + scol + 32, sraw + 32);
            tmem_ld32(tmem + lane_base + scol + 64, sraw + 64);
            tmem_ld32(tmem + lane_base + scol + 96, sraw + 96);
            tmem_wait_ld();

            const int n0 = j * BN;
            const bool need_mask = (n0 + BN > a.n_kv) || (a.causal && n0 + BN - 1 > m0 + offset) ||
                                   (a.key_mask != nullptr && n0 + BN > first_unkept);
            if (need_mask) {
                const uint8_t* km = a.key_mask ? a.key_mask + (size_t)b * a.n_kv : nullptr;
#pragma unroll
                for (int c = 0; c < BN; ++c) {
                    const int key = n0 + c;
                    bool keep = key < a.n_kv && key <= row_limit;
                    if (km != nullptr && keep) keep = km[key] != 0;
                    if (!keep) sraw[c] = 0xff800000u;  // -inf
                }
            }
            float mx = __uint_as_float(sraw[0]);
#pragma unroll
            for (int c = 1; c < BN; ++c) mx = fmaxf(mx, __uint_as_float(sraw[c]));
            const float m_new = fmaxf(m_run, mx * sl2);
            const float base = (m_new == -INFINITY) ? 0.f : m_new;
            const float alpha = ex2_approx(m_run - base);
            float sum = 0.f;
            uint32_t preg[BN / 2];
#pragma unroll
            for (int c = 0; c < BN; c += 2) {
                const float p0 = ex2_approx(fmaf(__uint_as_float(sraw[c]), sl2, -base));
                const float p1 = ex2_approx(fmaf(__uint_as_float(sraw[c + 1]), sl2, -base));
                sum += p0 + p1;
                preg[c / 2] = pack_bf16x2(p0, p1);
            }
            // O must hold every earlier P V before it is rescaled or P_j is handed over
            if (j >= 1) {
                if (!warp_wait(&bar.o_full, (j - 1) & 1, &bar.abort_flag, status, kSiteOFull)) { ok = false; break; }
                tc_fence_after();
                if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(tmem + lane_base + kColO + 32 * c, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32(tmem + lane_base + kColO + 32 * c, o);
                    }
                }
            }
            tmem_st32(tmem + lane_base + scol, preg);
            tmem_st32(tmem + lane_base + scol + 32, preg + 32);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bar.p_full[buf]);
            l_run = l_run * alpha + sum;
            m_run = m_new;
            if (tid == 0) trace_mark(trace, kTrSoftmax, (uint32_t)j + 1u);
        }

        // epilogue: O / l in bf16 and the log-sum-exp (natural log of the scaled scores)
        if (ok && n_blk > 0) {
            ok = warp_wait(&bar.o_full, (n_blk - 1) & 1, &bar.abort_flag, status, kSiteOFinal);
            tc_fence_after();
        }
        const bool has = ok && n_blk > 0 && l_run > 0.f;
        const float inv = has ? 1.f / l_run : 0.f;
        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.o) + ((size_t)(b * a.H + h) * a.n_q + row) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            if (ok && n_blk > 0) {
                tmem_ld32(tmem + lane_base + kColO + 32 * c, o);
                tmem_wait_ld();
            }
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
                w[e] = has ? pack_bf16x2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv) : 0u;
            if (row < a.n_q) {
                uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
                for (int e = 0; e < 4; ++e) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
            }
        }
        if (a.lse != nullptr && row < a.n_q)
            a.lse[(size_t)(b * a.H + h) * a.n_q + row] =
                has ? (m_run + log2f(l_run)) * 0.6931471805599453f : -INFINITY;
        if (tid == 0) trace_mark(trace, kTrEpilogue, 1);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
        if (tid % 32 == 0) trace_mark(trace, kTrExit, 1);
    }
}

template <int D>
cudaError_t launch_d(const FwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     unsigned int* status, cudaStream_t stream) {
    // at least ~116 KB so that one CTA (and one 512-column TMEM allocation) sits on each SM
    const int smem = std::max(Layout<D>::kBytes + 1024, 118 * 1024);
    cudaError_t e = cudaFuncSetAttribute(fwd_bf16_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    // each CTA allocates all 512 TMEM columns, so exactly one may be resident per SM
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fwd_bf16_kernel<D>, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm != 1) return cudaErrorInvalidConfiguration;
    dim3 grid((a.n_q + BM - 1) / BM, a.H, a.B);
    fwd_bf16_kernel<D><<<grid, kThreads, smem, stream>>>(tq, tk, tv, a, status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_bf16_sm100(const FwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                                  const CUtensorMap& tv, unsigned int* status, cudaStream_t stream) {
    switch (a.d) {
        case 64: return launch_d<64>(a, tq, tk, tv, status, stream);
        case 128: return launch_d<128>(a, tq, tk, tv, status, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace attn
