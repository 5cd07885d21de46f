// Backward pass of exact attention with recomputation: dQ, dK, dV from Q, K, V,
// O, dO and the forward's log-sum-exp, without the n x n weight matrix in memory
// ("Dialogo con Gemini", section "Ricalcolo nel Backward Pass (Recomputation)":
// only the row statistics are kept, and the score and weight blocks are
// recomputed tile by tile on chip).  For one query head and its kept keys:
//
//   P_ij  = exp(scale q_i.k_j - LSE_i)        (the forward's LSE normalises P)
//   dV_j += sum_i P_ij dO_i
//   dS_ij = P_ij (dO_i.v_j - dO_i.O_i)        (sum_k P_ik dP_ik = dO_i.O_i)
//   dQ_i  = scale sum_j dS_ij k_j
//   dK_j += scale sum_i dS_ij q_i              (dK, dV summed over the group's query heads)
//
// Three kernels, all deterministic (no atomics):
//   bwd_prep_kernel   one warp per query row: dO.O and LSE * log2(e) into a
//                     workspace padded to 64 rows per head (pad rows: weight 0).
//   bwd_dkdv_kernel   one CTA per (64-key block, kv head, batch row); four warps,
//                     16 keys each, walk every query block of every query head of
//                     the group: S^T = K Q^T and dP^T = V dO^T, P and dS in
//                     registers, then dV += P^T dO and dK += dS^T Q with P and dS
//                     (bf16) as the A operands straight from the accumulators.
//   bwd_dq_kernel     one CTA per (64-query block, head, batch row); four warps,
//                     16 queries each, walk the key blocks: S = Q K^T, dP = dO V^T,
//                     dQ += dS K.
// The products run as mma.sync m16n8k16 (bf16 in, fp32 accumulate).  Tiles come
// in by TMA (128-byte swizzle, zero fill past the ends) through double-buffered
// shared memory, announced on mbarriers whose waits are bounded; a wait that
// gives up records the site in the status word and the CTA returns without
// writing.  Splitting dQ from dK/dV recomputes S and dP once more (7 products
// instead of 5) in exchange for no atomics and no cross-CTA reduction.
#include <algorithm>
#include <cmath>
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace attn {
namespace {

using namespace dev;

constexpr int kRows = 64;               // rows of every tile (keys or queries)
constexpr int kWarps = 4;               // 16 rows each
constexpr int kThreads = 32 * kWarps;
constexpr int kHalfBytes = kRows * 128;  // [64 rows][64 bf16], 128-byte swizzled
constexpr float kLog2e = 1.4426950408889634f;

enum : uint32_t { kSiteKV = 0x31, kSiteQD = 0x32, kSiteQ = 0x33, kSiteStep = 0x34 };

template <int D>
struct BwdTile {
    static constexpr int kHalves = D / 64;
    static constexpr int kBytes = kHalves * kHalfBytes;
};

// byte offset of 16-byte chunk c (0 .. D/8-1) of row r in a [D/64][64][64] swizzled tile
__device__ __forceinline__ uint32_t toff(int r, int c) {
    return (uint32_t)((c >> 3) * kHalfBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm4t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
// d += A B, m16n8k16, bf16 in, fp32 accumulate; a = {rows 0-7 k 0-7, rows 8-15 k 0-7, rows 0-7 k 8-15,
// rows 8-15 k 8-15}, b = {k 0-7, k 8-15}
__device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// A fragment (16 rows x 16 k) at rows r0.., k chunk pair kc (columns 16 kc ..) of a row-major tile.
__device__ __forceinline__ void load_a(uint32_t tile, int r0, int kc, int lane, uint32_t (&a)[4]) {
    ldsm4(tile + toff(r0 + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * kc + (lane >> 4)), a);
}
// B fragments of two 8-column n-tiles (rows n0 .. n0+15 of a tile stored [n][k]) at k chunk pair kc:
// b[0], b[1] for n-tile 0 and b[2], b[3] for n-tile 1.
__device__ __forceinline__ void load_b_nk(uint32_t tile, int n0, int kc, int lane, uint32_t (&b)[4]) {
    ldsm4(tile + toff(n0 + (lane & 7) + (lane >> 4) * 8, 2 * kc + ((lane >> 3) & 1)), b);
}
// The same for a tile stored [k][n] (k = rows k0 .. k0+15, n = columns 16 nc ..), transposed on load.
__device__ __forceinline__ void load_b_kn(uint32_t tile, int k0, int nc, int lane, uint32_t (&b)[4]) {
    ldsm4t(tile + toff(k0 + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * nc + (lane >> 4)), b);
}

// Rows [16 w, 16 w + 16) of S = A B^T for a 64-column B, both [rows][D] tiles: acc[nt] holds columns 8 nt ..
template <int D>
__device__ __forceinline__ void rows_times_tile(uint32_t a_tile, uint32_t b_tile, int r0, int lane,
                                                float (&acc)[8][4]) {
#pragma unroll
    for (int kc = 0; kc < D / 16; ++kc) {
        uint32_t a[4];
        load_a(a_tile, r0, kc, lane, a);
#pragma unroll
        for (int np = 0; np < 4; ++np) {
            uint32_t b[4];
            load_b_nk(b_tile, 16 * np, kc, lane, b);
            mma(acc[2 * np], a, b[0], b[1]);
            mma(acc[2 * np + 1], a, b[2], b[3]);
        }
    }
}

// acc (16 x D) += X (16 x 64, in registers as bf16 A fragments) * T (64 x D tile stored [k][n])
template <int D>
__device__ __forceinline__ void regs_times_tile(const uint32_t (&x)[4][4], uint32_t tile, int lane,
                                                float (&acc)[D / 8][4]) {
#pragma unroll
    for (int kq = 0; kq < 4; ++kq) {
#pragma unroll
        for (int nc = 0; nc < D / 16; ++nc) {
            uint32_t b[4];
            load_b_kn(tile, 16 * kq, nc, lane, b);
            mma(acc[2 * nc], x[kq], b[0], b[1]);
            mma(acc[2 * nc + 1], x[kq], b[2], b[3]);
        }
    }
}

// Accumulator tiles (16 x 64 as 8 n-tiles) to bf16 A fragments over k = the 64 columns.
__device__ __forceinline__ void to_a_frags(const float (&c)[8][4], uint32_t (&x)[4][4]) {
#pragma unroll
    for (int kq = 0; kq < 4; ++kq) {
        x[kq][0] = pack_bf16x2(c[2 * kq][0], c[2 * kq][1]);
        x[kq][1] = pack_bf16x2(c[2 * kq][2], c[2 * kq][3]);
        x[kq][2] = pack_bf16x2(c[2 * kq + 1][0], c[2 * kq + 1][1]);
        x[kq][3] = pack_bf16x2(c[2 * kq + 1][2], c[2 * kq + 1][3]);
    }
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

template <int D>
__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int row0, int head,
                                          int batch) {
#pragma unroll
    for (int hf = 0; hf < D / 64; ++hf) tma_load_4d(dst + hf * kHalfBytes, map, bar, hf * 64, row0, head, batch);
}

// Let copies still landing in shared memory finish before an aborting CTA exits:
// steps [from, issued) of a two-buffer ring.
__device__ __forceinline__ void drain_ring(uint64_t* ring, int from, int issued) {
    for (int s = from; s < issued; ++s) mbar_drain(&ring[s & 1], (s >> 1) & 1);
}

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

template <int D>
struct DkdvSmem {
    static constexpr int kT = BwdTile<D>::kBytes;
    static constexpr int kOffK = 0, kOffV = kT, kOffQ = 2 * kT, kOffO = 4 * kT;  // Q[2], dO[2]
    static constexpr int kOffL = 6 * kT;                  // float l2[2][64], dd[2][64]
    static constexpr int kOffBar = kOffL + 4 * kRows * 4;  // kv_full, qd_full[2], abort flag
    static constexpr int kBytes = kOffBar + 64;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                    const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo, const BwdArgs a,
                    unsigned int* status) {
    using L = DkdvSmem<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float* s_l2 = reinterpret_cast<float*>(smem + L::kOffL);   // [2][64]
    float* s_dd = s_l2 + 2 * kRows;                            // [2][64]
    uint64_t* kv_full = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
    uint64_t* qd_full = kv_full + 1;                           // [2]
    volatile int* abort_flag = reinterpret_cast<volatile int*>(kv_full + 3);

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int n_kb = (a.n_kv + kRows - 1) / kRows;
    const int per = a.H_kv * a.B;
    const int kb = blockIdx.x / per;          // heaviest key blocks (the first, under a causal mask) first
    const int g = (blockIdx.x % per) % a.H_kv, b = (blockIdx.x % per) / a.H_kv;
    if (kb >= n_kb) return;
    const int j0 = kb * kRows;
    const int group = a.H / a.H_kv;
    const int off = a.n_kv - a.n_q;           // key j is visible to query i when j <= i + off (causal)
    const int n_qb = (a.n_q + kRows - 1) / kRows;
    const int qb0 = a.causal ? max(0, j0 - off) / kRows : 0;
    const int per_head = n_qb - qb0;
    const int steps = group * per_head;

    if (tid == 0) {
        mbar_init(kv_full, 1);
        mbar_init(&qd_full[0], 1);
        mbar_init(&qd_full[1], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const size_t l_stride = (size_t)a.n_q_pad;
    auto issue_step = [&](int t) {
        const int buf = t & 1;
        const int h = g * group + t / per_head, qb = qb0 + t % per_head;
        mbar_arrive_expect_tx(&qd_full[buf], 2 * L::kT + 2 * kRows * 4);
        load_tile<D>(smem + L::kOffQ + buf * L::kT, &tq, &qd_full[buf], qb * kRows, h, b);
        load_tile<D>(smem + L::kOffO + buf * L::kT, &tdo, &qd_full[buf], qb * kRows, h, b);
        const size_t row0 = ((size_t)b * a.H + h) * l_stride + (size_t)qb * kRows;
        bulk_load(s_l2 + buf * kRows, a.ws_l2 + row0, kRows * 4, &qd_full[buf]);
        bulk_load(s_dd + buf * kRows, a.ws_dd + row0, kRows * 4, &qd_full[buf]);
    };
    int issued = 0;   // steps whose copies thread 0 has requested
    if (tid == 0) {
        mbar_arrive_expect_tx(kv_full, 2 * L::kT);
        load_tile<D>(smem + L::kOffK, &tk, kv_full, j0, g, b);
        load_tile<D>(smem + L::kOffV, &tv, kv_full, j0, g, b);
        issue_step(0);
        issued = 1;
    }
    const uint32_t sK = smem_u32(smem + L::kOffK), sV = smem_u32(smem + L::kOffV);

    // this thread's two key rows (accumulator rows lane/4 and lane/4 + 8 of its warp)
    const int jr0 = j0 + warp * 16 + lane / 4, jr1 = jr0 + 8;
    const bool key0 = jr0 < a.n_kv && (a.key_mask == nullptr || a.key_mask[(size_t)b * a.n_kv + jr0] != 0);
    const bool key1 = jr1 < a.n_kv && (a.key_mask == nullptr || a.key_mask[(size_t)b * a.n_kv + jr1] != 0);
    const float c = a.scale * kLog2e;

    float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) dk[i][e] = dv[i][e] = 0.f;

    bool ok = __syncthreads_and(mbar_wait(kv_full, 0, abort_flag, status, kSiteKV));
    int t = 0;
    for (; ok && t < steps; ++t) {
        const int buf = t & 1;
        if (tid == 0 && t + 1 < steps) {
            issue_step(t + 1);
            issued = t + 2;
        }
        ok = __syncthreads_and(mbar_wait(&qd_full[buf], (t >> 1) & 1, abort_flag, status, kSiteQD));
        if (!ok) break;
        const uint32_t sQ = smem_u32(smem + L::kOffQ + buf * L::kT);
        const uint32_t sO = smem_u32(smem + L::kOffO + buf * L::kT);
        const int i0 = (qb0 + t % per_head) * kRows;

        float s[8][4], dp[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[nt][e] = dp[nt][e] = 0.f;
        rows_times_tile<D>(sK, sQ, warp * 16, lane, s);   // S^T: keys x queries
        rows_times_tile<D>(sV, sO, warp * 16, lane, dp);  // dP^T
        const bool diag = a.causal && (j0 + kRows - 1 > i0 + off);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int col = nt * 8 + 2 * (lane % 4) + (e & 1);
                const int j = (e < 2) ? jr0 : jr1;
                bool keep = (e < 2) ? key0 : key1;
                if (diag) keep = keep && (j <= i0 + col + off);
                const float p = keep ? ex2_approx(fmaf(s[nt][e], c, -s_l2[buf * kRows + col])) : 0.f;
                s[nt][e] = p;
                dp[nt][e] = p * (dp[nt][e] - s_dd[buf * kRows + col]);
            }
        }
        uint32_t x[4][4];
        to_a_frags(s, x);
        regs_times_tile<D>(x, sO, lane, dv);   // dV += P^T dO
        to_a_frags(dp, x);
        regs_times_tile<D>(x, sQ, lane, dk);   // dK += dS^T Q
        __syncthreads();                        // buffer `buf` is refilled at step t + 2
    }
    if (!ok) {
        if (tid == 0) {
            mbar_drain(kv_full, 0);
            drain_ring(qd_full, t, issued);
        }
        return;
    }
    const int cq = 2 * (lane % 4);
    __nv_bfloat16* dk_out = static_cast<__nv_bfloat16*>(a.dk) + ((size_t)b * a.H_kv + g) * a.n_kv * D;
    __nv_bfloat16* dv_out = static_cast<__nv_bfloat16*>(a.dv) + ((size_t)b * a.H_kv + g) * a.n_kv * D;
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd) {
        if (jr0 < a.n_kv) {
            *reinterpret_cast<uint32_t*>(dk_out + (size_t)jr0 * D + nd * 8 + cq) =
                pack_bf16x2(dk[nd][0] * a.scale, dk[nd][1] * a.scale);
            *reinterpret_cast<uint32_t*>(dv_out + (size_t)jr0 * D + nd * 8 + cq) = pack_bf16x2(dv[nd][0], dv[nd][1]);
        }
        if (jr1 < a.n_kv) {
            *reinterpret_cast<uint32_t*>(dk_out + (size_t)jr1 * D + nd * 8 + cq) =
                pack_bf16x2(dk[nd][2] * a.scale, dk[nd][3] * a.scale);
            *reinterpret_cast<uint32_t*>(dv_out + (size_t)jr1 * D + nd * 8 + cq) = pack_bf16x2(dv[nd][2], dv[nd][3]);
        }
    }
}

template <int D>
struct DqSmem {
    static constexpr int kT = BwdTile<D>::kBytes;
    static constexpr int kOffQ = 0, kOffO = kT, kOffK = 2 * kT, kOffV = 4 * kT;  // K[2], V[2]
    static constexpr int kOffMask = 6 * kT;                 // uint8 key kept [2][64]
    static constexpr int kOffBar = kOffMask + 2 * kRows;    // q_full, kv_full[2], abort flag
    static constexpr int kBytes = kOffBar + 64;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo, const BwdArgs a,
                  unsigned int* status) {
    using L = DqSmem<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* s_keep = smem + L::kOffMask;                       // [2][64]
    uint64_t* q_full = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
    uint64_t* kv_full = q_full + 1;                             // [2]
    volatile int* abort_flag = reinterpret_cast<volatile int*>(q_full + 3);

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int n_qb = (a.n_q + kRows - 1) / kRows;
    const int per = a.H * a.B;
    const int qb = n_qb - 1 - (int)(blockIdx.x / per);   // heaviest query blocks (the last, when causal) first
    const int h = (blockIdx.x % per) % a.H, b = (blockIdx.x % per) / a.H;
    if (qb < 0) return;
    const int g = h / (a.H / a.H_kv);
    const int q0 = qb * kRows;
    const int off = a.n_kv - a.n_q;
    const int n_kb_all = (a.n_kv + kRows - 1) / kRows;
    int n_kb = n_kb_all;
    if (a.causal) {
        const int j_max = min(q0 + kRows, a.n_q) - 1 + off;   // last key any row of the block sees
        n_kb = j_max < 0 ? 0 : min(n_kb_all, j_max / kRows + 1);
    }

    if (tid == 0) {
        mbar_init(q_full, 1);
        mbar_init(&kv_full[0], 1);
        mbar_init(&kv_full[1], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    auto issue_kv = [&](int t) {
        const int buf = t & 1;
        mbar_arrive_expect_tx(&kv_full[buf], 2 * L::kT);
        load_tile<D>(smem + L::kOffK + buf * L::kT, &tk, &kv_full[buf], t * kRows, g, b);
        load_tile<D>(smem + L::kOffV + buf * L::kT, &tv, &kv_full[buf], t * kRows, g, b);
    };
    auto fill_keep = [&](int t) {   // plain stores, read after the step's barrier
        if (tid < kRows) {
            const int j = t * kRows + tid;
            s_keep[(t & 1) * kRows + tid] =
                j < a.n_kv && (a.key_mask == nullptr || a.key_mask[(size_t)b * a.n_kv + j] != 0);
        }
    };
    int issued = 0;   // key blocks whose copies thread 0 has requested
    if (tid == 0 && n_kb > 0) {
        mbar_arrive_expect_tx(q_full, 2 * L::kT);
        load_tile<D>(smem + L::kOffQ, &tq, q_full, q0, h, b);
        load_tile<D>(smem + L::kOffO, &tdo, q_full, q0, h, b);
        issue_kv(0);
        issued = 1;
    }
    if (n_kb > 0) fill_keep(0);
    const uint32_t sQ = smem_u32(smem + L::kOffQ), sO = smem_u32(smem + L::kOffO);

    const int ir0 = q0 + warp * 16 + lane / 4, ir1 = ir0 + 8;   // this thread's two query rows
    const size_t lrow = ((size_t)b * a.H + h) * a.n_q_pad;
    const float l2_0 = a.ws_l2[lrow + ir0], l2_1 = a.ws_l2[lrow + ir1];   // pad rows: +inf
    const float dd_0 = a.ws_dd[lrow + ir0], dd_1 = a.ws_dd[lrow + ir1];
    const float c = a.scale * kLog2e;

    float dq[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) dq[i][e] = 0.f;

    bool ok = true;
    if (n_kb > 0) ok = __syncthreads_and(mbar_wait(q_full, 0, abort_flag, status, kSiteQ));
    int t = 0;
    for (; ok && t < n_kb; ++t) {
        const int buf = t & 1;
        if (t + 1 < n_kb) {
            if (tid == 0) {
                issue_kv(t + 1);
                issued = t + 2;
            }
            fill_keep(t + 1);
        }
        ok = __syncthreads_and(mbar_wait(&kv_full[buf], (t >> 1) & 1, abort_flag, status, kSiteStep));
        if (!ok) break;
        const uint32_t sK = smem_u32(smem + L::kOffK + buf * L::kT);
        const uint32_t sV = smem_u32(smem + L::kOffV + buf * L::kT);
        const int j0 = t * kRows;

        float s[8][4], dp[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[nt][e] = dp[nt][e] = 0.f;
        rows_times_tile<D>(sQ, sK, warp * 16, lane, s);    // S: queries x keys
        rows_times_tile<D>(sO, sV, warp * 16, lane, dp);   // dP
        const bool diag = a.causal && (j0 + kRows - 1 > q0 + off);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int col = nt * 8 + 2 * (lane % 4) + (e & 1);
                const int i = (e < 2) ? ir0 : ir1;
                bool keep = s_keep[buf * kRows + col] != 0;
                if (diag) keep = keep && (j0 + col <= i + off);
                const float p = keep ? ex2_approx(fmaf(s[nt][e], c, -((e < 2) ? l2_0 : l2_1))) : 0.f;
                dp[nt][e] = p * (dp[nt][e] - ((e < 2) ? dd_0 : dd_1));
            }
        }
        uint32_t x[4][4];
        to_a_frags(dp, x);
        regs_times_tile<D>(x, sK, lane, dq);   // dQ += dS K
        __syncthreads();                        // buffer `buf` is refilled at step t + 2
    }
    if (!ok) {
        if (tid == 0) {
            mbar_drain(q_full, 0);
            drain_ring(kv_full, t, issued);
        }
        return;
    }
    const int cq = 2 * (lane % 4);
    __nv_bfloat16* dq_out = static_cast<__nv_bfloat16*>(a.dq) + ((size_t)b * a.H + h) * a.n_q * D;
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd) {
        if (ir0 < a.n_q)
            *reinterpret_cast<uint32_t*>(dq_out + (size_t)ir0 * D + nd * 8 + cq) =
                pack_bf16x2(dq[nd][0] * a.scale, dq[nd][1] * a.scale);
        if (ir1 < a.n_q)
            *reinterpret_cast<uint32_t*>(dq_out + (size_t)ir1 * D + nd * 8 + cq) =
                pack_bf16x2(dq[nd][2] * a.scale, dq[nd][3] * a.scale);
    }
}

template <int D>
cudaError_t launch_d(const BwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const CUtensorMap& tdo, unsigned int* status, cudaStream_t stream) {
    const int smem_kv = DkdvSmem<D>::kBytes + 1024, smem_q = DqSmem<D>::kBytes + 1024;
    cudaError_t e = cudaFuncSetAttribute(bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_kv);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_q);
    if (e != cudaSuccess) return e;
    const long long n_kb = (a.n_kv + kRows - 1) / kRows, n_qb = (a.n_q + kRows - 1) / kRows;
    const long long grid_kv = n_kb * a.H_kv * a.B, grid_q = n_qb * a.H * a.B;
    if (grid_kv > 0x7fffffffll || grid_q > 0x7fffffffll) return cudaErrorInvalidConfiguration;
    bwd_dkdv_kernel<D><<<(unsigned)grid_kv, kThreads, smem_kv, stream>>>(tq, tk, tv, tdo, a, status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    bwd_dq_kernel<D><<<(unsigned)grid_q, kThreads, smem_q, stream>>>(tq, tk, tv, tdo, a, status);
    return cudaGetLastError();
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
