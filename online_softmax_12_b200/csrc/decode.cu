// Paged split-KV decode and the merge of its partial states.
//
// Decode: one query token per sequence reads the whole KV cache of that
// sequence, so the work is bound by HBM bandwidth ("attention_matrix_deep",
// prefill vs decode: the matrix degenerates to a 1 x n vector and reading K and
// V is the bottleneck).  The cache is paged: fixed-size blocks and a block table
// that maps logical positions to physical pages ("Kernel di attenzione rapida e
// fusione degli operatori", section "Attenzione di tipo FlashAttention e
// attenzione paginata").
//
// Kernel 1, one CTA per (split c, kv head g, sequence s): tokens
// [c*T, min((c+1)*T, len_s)) of that sequence, for the G query heads that share
// kv head g.  Each token row (D bf16 = D*2 bytes) is read by D/8 lanes with one
// 16-byte load each, so a warp covers 32*16 contiguous bytes per load step.
// Every group of D/8 lanes keeps, per query head, the running (m, l, u) state of
// "Attenzione: softmax online, riscalamento e memoria", section 2, updated a
// chunk of tokens at a time (one rescale per chunk).  The groups' states are
// merged in shared memory and written as one fp32 partial (m, l, u) per head.
//
// This file holds the CUDA-core variant (any page size) and the merge; the
// tensor-core variant for 16-token pages is in decode_mma.cu.
//
// Kernel 2, one CTA per (sequence, query head): merges the partials of all
// splits with the disjoint-set rule of section 4 (rescale every part to the
// largest m, then add), in a fixed order, and writes O = U / L and the
// log-sum-exp.
//
// Scores are kept in base-2 units (q pre-multiplied by scale * log2(e)) so every
// exponential is one ex2 instruction; the log-sum-exp is converted back to the
// natural log of the scaled scores on output.
#include <cmath>
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace attn {
namespace {

constexpr int kThreads = 128;
constexpr int kChunk = 4;  // tokens per lane group between rescales

__device__ __forceinline__ void bf16x8_to_f32(const uint4& w, float (&f)[8]) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(u[i] << 16);
        f[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
    }
}

template <int D, int G>
__global__ void __launch_bounds__(kThreads) decode_split_kernel(DecodeArgs a, unsigned int* status) {
    constexpr int LPT = D / 8;              // lanes per token row
    constexpr int NGRP = kThreads / LPT;    // lane groups per CTA
    __shared__ float sh_m[NGRP][G];
    __shared__ float sh_l[NGRP][G];
    __shared__ float sh_u[NGRP][G][D];

    const int c = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
    const int tid = threadIdx.x;
    const int grp = tid / LPT, lane = tid % LPT;

    int len = a.seq_lens[s];
    if (len < 0 || len > a.max_seq_len || len > a.max_pages * a.page_size) {
        if (tid == 0 && c == 0 && g == 0) atomicOr(status, ATTN_DEV_BAD_LEN);
        len = len < 0 ? 0 : min(len, min(a.max_seq_len, a.max_pages * a.page_size));
    }
    const int t_begin = c * a.split_tokens;
    if (t_begin >= len) return;  // the merge only reads splits that hold tokens
    const int t_end = min(t_begin + a.split_tokens, len);

    const float qscale = a.scale * 1.4426950408889634f;  // scores in log2 units
    float qf[G][8];
    const __nv_bfloat16* qp = static_cast<const __nv_bfloat16*>(a.q);
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
        const uint4 w = *reinterpret_cast<const uint4*>(qp + ((size_t)s * a.H + g * G + gi) * D + lane * 8);
        bf16x8_to_f32(w, qf[gi]);
#pragma unroll
        for (int e = 0; e < 8; ++e) qf[gi][e] *= qscale;
    }

    float m[G], l[G], u[G][8];
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
        m[gi] = -INFINITY;
        l[gi] = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) u[gi][e] = 0.f;
    }

    const __nv_bfloat16* kp = static_cast<const __nv_bfloat16*>(a.k_pages);
    const __nv_bfloat16* vp = static_cast<const __nv_bfloat16*>(a.v_pages);
    const int32_t* bt = a.block_table + (size_t)s * a.max_pages;
    const size_t tok_stride = (size_t)a.H_kv * D;  // elements between slots of a page

    // The trip count must be the same for every lane of a warp (the score
    // reduction below shuffles across the whole warp), so the loop runs over
    // warp-sized slabs of GPW lane groups and masks tokens past t_end.
    constexpr int GPW = 32 / LPT;          // lane groups per warp
    constexpr int kWarps = kThreads / 32;
    const int sub = (tid % 32) / LPT;      // this lane group within its warp
    for (int slab = t_begin + (tid / 32) * GPW * kChunk; slab < t_end; slab += kWarps * GPW * kChunk) {
        const int t0 = slab + sub * kChunk;
        uint4 kw[kChunk], vw[kChunk];
        bool ok[kChunk];
#pragma unroll
        for (int i = 0; i < kChunk; ++i) {
            const int t = t0 + i;
            ok[i] = t < t_end;
            if (ok[i]) {
                const int page = bt[t / a.page_size];
                if (page < 0 || page >= a.num_pages) {
                    ok[i] = false;
                    atomicOr(status, ATTN_DEV_BAD_PAGE);
                } else {
                    const size_t off = ((size_t)page * a.page_size + (t % a.page_size)) * tok_stride +
                                       (size_t)g * D + lane * 8;
                    kw[i] = __ldg(reinterpret_cast<const uint4*>(kp + off));
                    vw[i] = __ldg(reinterpret_cast<const uint4*>(vp + off));
                }
            }
        }
        // scores of the chunk, reduced over the LPT lanes of the token row
        float sc[kChunk][G];
#pragma unroll
        for (int i = 0; i < kChunk; ++i) {
            float kf[8];
            bf16x8_to_f32(ok[i] ? kw[i] : make_uint4(0, 0, 0, 0), kf);
#pragma unroll
            for (int gi = 0; gi < G; ++gi) {
                float acc = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) acc = fmaf(qf[gi][e], kf[e], acc);
                sc[i][gi] = acc;
            }
        }
#pragma unroll
        for (int off = LPT / 2; off >= 1; off >>= 1)
#pragma unroll
            for (int i = 0; i < kChunk; ++i)
#pragma unroll
                for (int gi = 0; gi < G; ++gi) sc[i][gi] += __shfl_xor_sync(0xffffffffu, sc[i][gi], off);

#pragma unroll
        for (int gi = 0; gi < G; ++gi) {
            float cmax = -INFINITY;
#pragma unroll
            for (int i = 0; i < kChunk; ++i)
                if (ok[i]) cmax = fmaxf(cmax, sc[i][gi]);
            const float m_new = fmaxf(m[gi], cmax);
            const float base = (m_new == -INFINITY) ? 0.f : m_new;
            const float alpha = dev::ex2_approx(m[gi] - base);
            l[gi] *= alpha;
#pragma unroll
            for (int e = 0; e < 8; ++e) u[gi][e] *= alpha;
            m[gi] = m_new;
#pragma unroll
            for (int i = 0; i < kChunk; ++i) {
                const float p = ok[i] ? dev::ex2_approx(sc[i][gi] - base) : 0.f;
                l[gi] += p;
                float vf[8];
                bf16x8_to_f32(ok[i] ? vw[i] : make_uint4(0, 0, 0, 0), vf);
#pragma unroll
                for (int e = 0; e < 8; ++e) u[gi][e] = fmaf(p, vf[e], u[gi][e]);
            }
        }
    }

    // merge the lane groups' states (section 4 rule) and write one partial per head
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
        if (lane == 0) {
            sh_m[grp][gi] = m[gi];
            sh_l[grp][gi] = l[gi];
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) sh_u[grp][gi][lane * 8 + e] = u[gi][e];
    }
    __syncthreads();
    for (int idx = tid; idx < G * D; idx += kThreads) {
        const int gi = idx / D, col = idx % D;
        float M = -INFINITY;
        for (int k = 0; k < NGRP; ++k) M = fmaxf(M, sh_m[k][gi]);
        const float base = (M == -INFINITY) ? 0.f : M;
        float L = 0.f, U = 0.f;
        for (int k = 0; k < NGRP; ++k) {
            const float f = dev::ex2_approx(sh_m[k][gi] - base);
            L = fmaf(sh_l[k][gi], f, L);
            U = fmaf(sh_u[k][gi][col], f, U);
        }
        const size_t slot = ((size_t)s * a.H + g * G + gi) * a.n_splits + c;
        a.part_u[slot * D + col] = U;
        if (col == 0) {
            // (m, l for the log-sum-exp, l that normalises u): the same sum here
            a.part_ml[slot * 4 + 0] = M;
            a.part_ml[slot * 4 + 1] = L;
            a.part_ml[slot * 4 + 2] = L;
            a.part_ml[slot * 4 + 3] = 0.f;
        }
    }
}

// Merge of the partial states of all splits of one (sequence, query head): the
// disjoint-set rule of section 4, in split order.  Each partial carries m (base 2),
// the exact weight sum (for the log-sum-exp) and the sum of the weights its
// accumulator actually used (which normalises O).
template <int D>
__global__ void __launch_bounds__(D) decode_merge_kernel(DecodeArgs a) {
    // launched as a programmatic dependent of the split kernel: its start-up overlaps the
    // split kernel's tail, and this wait returns once the partial states are complete
    dev::grid_dependency_wait();
    const int h = blockIdx.x, s = blockIdx.y;
    const int col = threadIdx.x;
    int len = a.seq_lens[s];
    len = len < 0 ? 0 : min(len, min(a.max_seq_len, a.max_pages * a.page_size));
    const int n_used = (len + a.split_tokens - 1) / a.split_tokens;
    const size_t slot0 = ((size_t)s * a.H + h) * a.n_splits;
    // one pass in split order: the running maximum M and the sums measured against it
    // (the same rescale as within a split), so the loads of several splits are in
    // flight together instead of one dependent pass for the maximum and another for
    // the sums
    float M = -INFINITY, Le = 0.f, Lo = 0.f, U = 0.f;
#pragma unroll 4
    for (int c = 0; c < n_used; ++c) {
        const float4 ml = *reinterpret_cast<const float4*>(a.part_ml + (slot0 + c) * 4);
        const float u = a.part_u[(slot0 + c) * D + col];
        const float Mn = fmaxf(M, ml.x);
        const float base = (Mn == -INFINITY) ? 0.f : Mn;
        const float f_old = dev::ex2_approx(M - base), f_new = dev::ex2_approx(ml.x - base);
        Le = fmaf(Le, f_old, ml.y * f_new);
        Lo = fmaf(Lo, f_old, ml.z * f_new);
        U = fmaf(U, f_old, u * f_new);
        M = Mn;
    }
    const float out = (Lo > 0.f) ? U / Lo : 0.f;
    static_cast<__nv_bfloat16*>(a.o)[((size_t)s * a.H + h) * D + col] = __float2bfloat16_rn(out);
    if (a.lse != nullptr && col == 0)
        a.lse[(size_t)s * a.H + h] = (Le > 0.f) ? (M + log2f(Le)) * 0.6931471805599453f : -INFINITY;
}

template <int D, int G>
cudaError_t launch_dg(const DecodeArgs& a, unsigned int* status, cudaStream_t stream) {
    dim3 grid(a.n_splits, a.H_kv, a.num_seqs);
    decode_split_kernel<D, G><<<grid, kThreads, 0, stream>>>(a, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_decode_merge(a, stream);
}

template <int D>
cudaError_t launch_d(const DecodeArgs& a, unsigned int* status, cudaStream_t stream) {
    switch (a.H / a.H_kv) {
        case 1: return launch_dg<D, 1>(a, status, stream);
        case 2: return launch_dg<D, 2>(a, status, stream);
        case 4: return launch_dg<D, 4>(a, status, stream);
        case 8: return launch_dg<D, 8>(a, status, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_decode_merge(const DecodeArgs& a, cudaStream_t stream) {
    if (a.num_seqs == 0) return cudaSuccess;
    if (a.d != 64 && a.d != 128) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.H, a.num_seqs, 1);
    cfg.blockDim = dim3(a.d, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = a.d == 64 ? cudaLaunchKernelEx(&cfg, decode_merge_kernel<64>, a)
                              : cudaLaunchKernelEx(&cfg, decode_merge_kernel<128>, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs& a, unsigned int* status, cudaStream_t stream) {
    if (a.num_seqs == 0) return cudaSuccess;
    switch (a.d) {
        case 64: return launch_d<64>(a, status, stream);
        case 128: return launch_d<128>(a, status, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace attn
