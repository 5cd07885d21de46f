// Paged split-KV decode on the tensor cores, for 16-token pages.
//
// Same computation as decode.cu's CUDA-core kernel (one query token per
// sequence, keys and values gathered page by page through the block table:
// "Kernel di attenzione rapida e fusione degli operatori", section
// "Attenzione di tipo FlashAttention e attenzione paginata"; the running
// (m, l, u) state of "Attenzione: softmax online, riscalamento e memoria",
// section 2, per query head; one fp32 partial per split for the merge of
// section 4), laid out so that HBM, not instruction issue, is the bound:
//
//   warp 4      producer: lane l owns ring stage l and copies pages l, l + 8, ...:
//               it reads the page id, checks it against the pool, and copies the page's K and
//               V rows for this kv head into an 8-stage shared-memory ring
//               with TMA (one 2 KB box of 16 slots x 64 columns per half row,
//               128-byte swizzle); a bad page id is skipped and reported.
//   warps 0-3   consumers: warp w takes pages w, w+4, ...; for each page
//               S = Q K^T and O += P V run as mma.sync m16n8k16 (bf16 in, fp32
//               accumulate) with the G query heads of the group as the rows
//               (rows G..15 are zero), K and V fragments from ldmatrix (V
//               transposed), the online softmax on the score fragments.
// The four consumer states are merged in shared memory and written as one
// partial (m, l for the log-sum-exp, l for the output, u) per head.
//
// Single-launch variant (kCluster): the C CTAs of one (sequence, kv head) form a
// thread-block cluster and split the sequence's pages into C contiguous shares.
// Each keeps its partial state in its own shared memory; after a cluster barrier
// every CTA merges a 1/C slice of the output columns, reading the C partials
// through distributed shared memory in rank order (the same section-4 rule and the
// same fixed order as the merge kernel), and writes O and the LSE.  A second
// barrier keeps every CTA's shared memory alive until its peers have read it.  No
// partial state reaches global memory and no second kernel is launched.
//
// Slots past the sequence end (or in a skipped page) are excluded by setting
// their scores to -inf and their V rows to zero, so whatever bits they hold
// (the pool's unused slots may be NaN) cannot reach the output through 0 * NaN.
#include <cmath>
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace attn {
namespace {

using namespace dev;

constexpr int kPage = 16;          // tokens per page (= rows of one MMA K block)
constexpr int kConsumers = 4;
constexpr int kThreads = 32 * (kConsumers + 1);
constexpr int kStages = 8;         // multiple of kConsumers: stage i % kStages always serves warp i % 4
constexpr int kHalfBytes = kPage * 128;  // [16 slots][64 bf16], 128-byte swizzled
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kTau = 8.0f;       // move the reference only when the maximum passes it by more
static_assert(kStages % kConsumers == 0, "stage ownership");

template <int D>
struct DecLayout {
    static constexpr int kHalves = D / 64;
    static constexpr int kStageBytes = 2 * kHalves * kHalfBytes;  // K halves, then V halves
    static constexpr int kOffStages = 0;
    static constexpr int kOffMerge = kStages * kStageBytes;
};
constexpr int kMaxCluster = 8;   // CTAs per (sequence, kv head) in the single-launch variant

struct DecBars {
    uint64_t full[kStages], empty[kStages];
    int page_ok[kStages];
    int abort_flag;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
// D = A B + D, m16n8k16, bf16 inputs, fp32 accumulators; A rows 8..15 (a1, a3) are zero here.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}
// byte address of 16-byte chunk `chunk` of row `row` in a 128-byte-swizzled [rows][64 bf16] half tile
__device__ __forceinline__ uint32_t swz(uint32_t half_base, int row, int chunk) {
    return half_base + row * 128 + ((chunk ^ (row & 7)) << 4);
}

// Three CTAs per SM (about 75 KB of shared memory each): 24 ring stages, 192 KB of
// K/V copies, can be in flight per SM, which HBM latency needs.
template <int D, int G, bool kCluster>
__global__ void __launch_bounds__(kThreads, 3)
    decode_mma_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                      const DecodeArgs a, unsigned int* status) {
    using L = DecLayout<D>;
    constexpr int H2 = L::kHalves;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    float* merge_m = reinterpret_cast<float*>(smem + L::kOffMerge);   // [kConsumers][G]
    float* merge_le = merge_m + kConsumers * G;                        // [kConsumers][G]
    float* merge_lo = merge_le + kConsumers * G;                       // [kConsumers][G]
    float* merge_u = merge_lo + kConsumers * G;                        // [kConsumers][G][D]
    DecBars& bar = *reinterpret_cast<DecBars*>(merge_u + kConsumers * G * D);
    // single launch: this CTA's partial state, read by its cluster peers
    float* cpart_ml = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(&bar + 1) + 15) & ~uintptr_t(15));
                                                                          // [G][4]: m, l_e, l_o, pad (16-byte aligned)
    float* cpart_u = cpart_ml + 4 * G;                                    // [G][D]

    const int c = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;

    int len = a.seq_lens[s];
    if (len < 0 || len > a.max_seq_len || len > a.max_pages * kPage) {
        if (tid == 0 && c == 0 && g == 0) atomicOr(status, ATTN_DEV_BAD_LEN);
        len = len < 0 ? 0 : min(len, min(a.max_seq_len, a.max_pages * kPage));
    }
    int t_begin, t_end, page0, n_pages;
    if constexpr (kCluster) {
        // C contiguous shares of whole pages; a share may be empty, but its CTA still takes
        // part in both cluster barriers (with an empty partial state)
        const int C = (int)gridDim.x;
        const int total = (len + kPage - 1) / kPage;
        const int per = (total + C - 1) / C;
        page0 = min(c * per, total);
        n_pages = min(per, total - page0);
        t_begin = page0 * kPage;
        t_end = min(t_begin + n_pages * kPage, len);
    } else {
        t_begin = c * a.split_tokens;  // a multiple of kPage
        if (t_begin >= len) return;    // the merge only reads splits that hold tokens
        t_end = min(t_begin + a.split_tokens, len);
        page0 = t_begin / kPage;
        n_pages = (t_end - t_begin + kPage - 1) / kPage;
    }

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&bar.full[i], 1);
            mbar_init(&bar.empty[i], 1);
        }
        bar.abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const uint32_t stage0 = smem_u32(smem + L::kOffStages);

    if (warp == kConsumers) {
        // ------------------------------------------------ producer
        // Lane l (l < kStages) owns ring stage l: it copies pages l, l + kStages, ...,
        // reading each page id itself, so up to kStages pages are requested at once
        // instead of one after another from a single thread.
        if (lane == 0) {
            tma_prefetch_desc(&tk);
            tma_prefetch_desc(&tv);
        }
        __syncwarp();
        if (lane < kStages) {
            const int32_t* bt = a.block_table + (size_t)s * a.max_pages + page0;
            const int st = lane;
            int issued = 0;  // pages of this stage whose copies were issued
            for (int i = lane; i < n_pages; i += kStages) {
                const int page = bt[i];
                if (!mbar_wait(&bar.empty[st], ((i / kStages) & 1) ^ 1, &bar.abort_flag, status, 1)) break;
                const bool ok = page >= 0 && page < a.num_pages;
                bar.page_ok[st] = ok;
                if (ok) {
                    uint8_t* dst = smem + L::kOffStages + st * L::kStageBytes;
                    mbar_arrive_expect_tx(&bar.full[st], L::kStageBytes);
#pragma unroll
                    for (int h = 0; h < H2; ++h) {
                        tma_load_4d(dst + h * kHalfBytes, &tk, &bar.full[st], h * 64, g, 0, page);
                        tma_load_4d(dst + (H2 + h) * kHalfBytes, &tv, &bar.full[st], h * 64, g, 0, page);
                    }
                } else {
                    atomicOr(status, ATTN_DEV_BAD_PAGE);
                    mbar_arrive(&bar.full[st]);
                }
                ++issued;
            }
            if (bar.abort_flag && issued > 0)
                // an aborted CTA must not exit with its last copies still landing in shared memory
                mbar_drain(&bar.full[st], ((lane + (issued - 1) * kStages) / kStages) & 1);
        }
    } else {
        // ------------------------------------------------ consumers
        const int grp = lane >> 2, tig = lane & 3;  // fragment row (query head) and column pair
        const bool real = grp < G;
        const float sl2 = a.scale * kLog2e;
        // Q as the A operand, rows = the G heads of this kv group (rows >= G are zero)
        uint32_t qa0[D / 16], qa2[D / 16];
        {
            const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
                static_cast<const __nv_bfloat16*>(a.q) + ((size_t)s * a.H + g * G + (real ? grp : 0)) * D);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                qa0[k] = real ? qrow[(16 * k + 2 * tig) / 2] : 0u;
                qa2[k] = real ? qrow[(16 * k + 8 + 2 * tig) / 2] : 0u;
            }
        }
        float m_ref = -INFINITY, l_e = 0.f, l_o = 0.f;
        float o[D / 8][4];
#pragma unroll
        for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
        bool ok = true;

        for (int i = warp; i < n_pages; i += kConsumers) {
            const int st = i % kStages;
            if (!warp_wait(&bar.full[st], (i / kStages) & 1, &bar.abort_flag, status, 2)) { ok = false; break; }
            const uint32_t kbase = stage0 + st * L::kStageBytes;
            const uint32_t vbase = kbase + H2 * kHalfBytes;
            const int nv = bar.page_ok[st] ? min(kPage, t_end - (t_begin + i * kPage)) : 0;  // valid slots
            if (nv < kPage) {
                // zero the V rows of invalid slots (any bits may sit there)
                uint8_t* vrows = smem + L::kOffStages + st * L::kStageBytes + H2 * kHalfBytes;
                for (int e = lane; e < H2 * (kPage - nv) * 8; e += 32) {
                    const int h = e / ((kPage - nv) * 8), rem = e % ((kPage - nv) * 8);
                    *reinterpret_cast<uint4*>(vrows + h * kHalfBytes + (nv + rem / 8) * 128 + (rem % 8) * 16) =
                        make_uint4(0, 0, 0, 0);
                }
                __syncwarp();
            }
            // S = Q K^T for the page's 16 slots (two n-tiles of 8 tokens)
            float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                const int mi = lane >> 3, rr = lane & 7;
                const int token = rr + 8 * (mi >> 1);
                const int chunk = 2 * (k & 3) + (mi & 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(swz(kbase + (k >> 2) * kHalfBytes, token, chunk), b0, b1, b2, b3);
                mma16816(sc[0], qa0[k], qa2[k], b0, b1);
                mma16816(sc[1], qa0[k], qa2[k], b2, b3);
            }
            // this lane's scores: head grp, tokens 8*nt + 2*tig + {0, 1}
            float x[4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int tok = 8 * nt + 2 * tig + e;
                    x[2 * nt + e] = (tok < nv) ? sc[nt][e] * sl2 : -INFINITY;
                }
            float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const bool move = mx > m_ref + kTau;
            const float new_ref = move ? mx : m_ref;
            const float base = (new_ref == -INFINITY) ? 0.f : new_ref;
            const float alpha = move ? ex2_approx(m_ref - base) : 1.f;
            if (__any_sync(0xffffffffu, move)) {
#pragma unroll
                for (int n = 0; n < D / 8; ++n) {
                    o[n][0] *= alpha;
                    o[n][1] *= alpha;
                }
            }
            float p[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) p[e] = real ? ex2_approx(x[e] - base) : 0.f;
            const uint32_t pa0 = pack_bf16x2(p[0], p[1]);  // head grp, tokens 2tig, 2tig+1
            const uint32_t pa2 = pack_bf16x2(p[2], p[3]);  // head grp, tokens 8+2tig, 9+2tig
            l_e = l_e * alpha + ((p[0] + p[1]) + (p[2] + p[3]));
            l_o = l_o * alpha + ((__uint_as_float(pa0 << 16) + __uint_as_float(pa0 & 0xFFFF0000u)) +
                                 (__uint_as_float(pa2 << 16) + __uint_as_float(pa2 & 0xFFFF0000u)));
            m_ref = new_ref;
            // O += P V: V transposed by ldmatrix, two 8-column n-tiles per load
#pragma unroll
            for (int dd = 0; dd < D / 16; ++dd) {
                const int mi = lane >> 3, rr = lane & 7;
                const int token = rr + 8 * (mi & 1);
                const int chunk = 2 * (dd & 3) + (mi >> 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(swz(vbase + (dd >> 2) * kHalfBytes, token, chunk), b0, b1, b2, b3);
                mma16816(o[2 * dd], pa0, pa2, b0, b1);
                mma16816(o[2 * dd + 1], pa0, pa2, b2, b3);
            }
            if (nv < kPage) fence_proxy_async();  // generic writes above before the next TMA into this stage
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar.empty[st]);
        }
        // row sums over the four lanes of each head
        l_e += __shfl_xor_sync(0xffffffffu, l_e, 1);
        l_e += __shfl_xor_sync(0xffffffffu, l_e, 2);
        l_o += __shfl_xor_sync(0xffffffffu, l_o, 1);
        l_o += __shfl_xor_sync(0xffffffffu, l_o, 2);
        if (real) {
            if (tig == 0) {
                merge_m[warp * G + grp] = ok ? m_ref : -INFINITY;
                merge_le[warp * G + grp] = ok ? l_e : 0.f;
                merge_lo[warp * G + grp] = ok ? l_o : 0.f;
            }
            float* u = merge_u + (warp * G + grp) * D;
#pragma unroll
            for (int n = 0; n < D / 8; ++n) {
                u[8 * n + 2 * tig] = ok ? o[n][0] : 0.f;
                u[8 * n + 2 * tig + 1] = ok ? o[n][1] : 0.f;
            }
        }
    }
    __syncthreads();
    // merge the consumer warps (section 4 rule) into this split's partial state
    for (int idx = tid; idx < G * D; idx += kThreads) {
        const int gi = idx / D, col = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, merge_m[w * G + gi]);
        const float base = (M == -INFINITY) ? 0.f : M;
        float Le = 0.f, Lo = 0.f, U = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumers; ++w) {
            const float f = ex2_approx(merge_m[w * G + gi] - base);
            Le = fmaf(merge_le[w * G + gi], f, Le);
            Lo = fmaf(merge_lo[w * G + gi], f, Lo);
            U = fmaf(merge_u[(w * G + gi) * D + col], f, U);
        }
        if constexpr (kCluster) {
            cpart_u[gi * D + col] = U;
            if (col == 0) *reinterpret_cast<float4*>(cpart_ml + gi * 4) = make_float4(M, Le, Lo, 0.f);
        } else {
            const size_t slot = ((size_t)s * a.H + g * G + gi) * a.n_splits + c;
            a.part_u[slot * D + col] = U;
            if (col == 0) *reinterpret_cast<float4*>(a.part_ml + slot * 4) = make_float4(M, Le, Lo, 0.f);
        }
    }
    if constexpr (kCluster) {
        // every CTA of the cluster, aborted or not, reaches both barriers
        cluster_sync();
        const uint32_t C = gridDim.x, rank = cluster_ctarank();
        const int per_rank = D / (int)C;                       // output columns this CTA merges
        const uint32_t ml_local = smem_u32(cpart_ml), u_local = smem_u32(cpart_u);
        for (int idx = tid; idx < G * per_rank; idx += kThreads) {
            const int gi = idx / per_rank, col = (int)rank * per_rank + idx % per_rank;
            // one pass in rank order with a running maximum, as the merge kernel
            float M = -INFINITY, Le = 0.f, Lo = 0.f, U = 0.f;
            for (uint32_t cc = 0; cc < C; ++cc) {
                const uint32_t ml = cluster_map(ml_local, cc) + gi * 16;
                const float m_c = ld_cluster_f32(ml), le_c = ld_cluster_f32(ml + 4), lo_c = ld_cluster_f32(ml + 8);
                const float u_c = ld_cluster_f32(cluster_map(u_local, cc) + (gi * D + col) * 4);
                const float Mn = fmaxf(M, m_c);
                const float base = (Mn == -INFINITY) ? 0.f : Mn;
                const float f_old = ex2_approx(M - base), f_new = ex2_approx(m_c - base);
                Le = fmaf(Le, f_old, le_c * f_new);
                Lo = fmaf(Lo, f_old, lo_c * f_new);
                U = fmaf(U, f_old, u_c * f_new);
                M = Mn;
            }
            const size_t row = (size_t)s * a.H + g * G + gi;
            static_cast<__nv_bfloat16*>(a.o)[row * D + col] = __float2bfloat16_rn(Lo > 0.f ? U / Lo : 0.f);
            if (a.lse != nullptr && rank == 0 && col == 0)
                a.lse[row] = (Le > 0.f) ? (M + log2f(Le)) * 0.6931471805599453f : -INFINITY;
        }
        // the peers' shared memory stays allocated until every CTA has read it
        cluster_sync();
    } else {
        // this CTA's partial state is written: the merge kernel may be scheduled
        grid_dependents_launch();
    }
}

template <int D, int G>
cudaError_t launch_dg(const DecodeArgs& a, const CUtensorMap& tk, const CUtensorMap& tv, unsigned int* status,
                      cudaStream_t stream) {
    using L = DecLayout<D>;
    const int smem = L::kOffMerge + (3 * kConsumers * G + kConsumers * G * D) * 4 + (int)sizeof(DecBars) +
                     16 + (4 * G + G * D) * 4 + 1024;
    if (a.n_splits < 0) {
        // single launch: clusters of C CTAs per (sequence, kv head), C = -n_splits
        const int C = -a.n_splits;
        if (C < 1 || C > kMaxCluster || D % C != 0) return cudaErrorInvalidValue;
        auto kern = decode_mma_kernel<D, G, true>;
        static std::atomic<unsigned long long> ready_cluster{0};
        int dev = 0;
        cudaError_t e = setup_once_per_device(ready_cluster, &dev, [kern, smem](int) {
            return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        });
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(C, a.H_kv, a.num_seqs);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = C;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, kern, tk, tv, a, status);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    }
    static std::atomic<unsigned long long> ready{0};
    int dev = 0;
    cudaError_t e = setup_once_per_device(ready, &dev, [smem](int) {
        return cudaFuncSetAttribute(decode_mma_kernel<D, G, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    });
    if (e != cudaSuccess) return e;
    dim3 grid(a.n_splits, a.H_kv, a.num_seqs);
    decode_mma_kernel<D, G, false><<<grid, kThreads, smem, stream>>>(tk, tv, a, status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_decode_merge(a, stream);
}

template <int D>
cudaError_t launch_d(const DecodeArgs& a, const CUtensorMap& tk, const CUtensorMap& tv, unsigned int* status,
                     cudaStream_t stream) {
    switch (a.H / a.H_kv) {
        case 1: return launch_dg<D, 1>(a, tk, tv, status, stream);
        case 2: return launch_dg<D, 2>(a, tk, tv, status, stream);
        case 4: return launch_dg<D, 4>(a, tk, tv, status, stream);
        case 8: return launch_dg<D, 8>(a, tk, tv, status, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_decode_mma(const DecodeArgs& a, const CUtensorMap& tk, const CUtensorMap& tv,
                              unsigned int* status, cudaStream_t stream) {
    if (a.num_seqs == 0) return cudaSuccess;
    if (a.page_size != kPage || (a.n_splits > 0 && a.split_tokens % kPage != 0)) return cudaErrorInvalidValue;
    switch (a.d) {
        case 64: return launch_d<64>(a, tk, tv, status, stream);
        case 128: return launch_d<128>(a, tk, tv, status, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace attn
