// bf16 forward attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Method: the blocked online softmax ("Sviluppo AI ed Algebra Lineare",
// sections "Tiling" and "Online Softmax (La Formalizzazione Matematica)"; the
// (m, l, u) invariant of "Attenzione: softmax online, riscalamento e memoria",
// section 2).  For each 128-row query tile the kernel walks the key/value
// blocks; per block it forms S = Q K^T, updates the row maximum, the
// normaliser l and the unnormalised output u (in TMEM) and adds P V with
// P = 2^(S * scale * log2(e) - m_ref).  Normalisation by l happens once at the
// end (the deferred normalisation of the FlashAttention-2 section of the
// chat page), as does the log-sum-exp.
//
// The reference m_ref that u and l are measured against is only moved when the
// row maximum exceeds it by more than kTau (base 2): the invariant needs u and l
// to share one reference, not that the reference be the exact maximum (same
// page, sections 1-2), so P stays <= 2^kTau and most blocks skip the O rescale.
//
// B200 mapping: one CTA = two 128-row query tiles of one (batch, head), 12 warps.
//   warps 0-3, 4-7  softmax warpgroups, one per tile: thread t owns row t of its
//                   tile (TMEM lane t); loads the score row from TMEM, masks,
//                   takes the maximum, rescales its O row when the reference
//                   moves, writes P (bf16) over the first half of the same TMEM
//                   columns in two halves of 64 keys, each announced on its own
//                   barrier, and finally writes O / l and the LSE.
//   warp 8          TMEM allocator and single-thread tcgen05.mma issuer.
//   warps 9, 10     TMA producers: warp 9 each item's Q tiles and K_j, warp 10 V_j,
//                   each through a 2-stage shared-memory ring (128-byte swizzle,
//                   expect_tx); with paged keys and values eight lanes copy a block's
//                   eight pages.
//   warp 11         idle (it completes the third warpgroup for the register split).
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D, 256+2D).
// The MMA order per key block j is  PV0_j, S0_{j+1}, PV1_j, S1_{j+1}: while one
// warpgroup computes its softmax the tensor core works on the other tile, and
// because S_i_{j+1} is issued after PV_i_j, its completion also proves that
// P_i_j has been consumed and O_i is quiescent.  PV_i_j is issued in two halves
// of 64 keys, the first while the softmax still exponentiates the second.
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
constexpr int kTiles = 2;        // query tiles per CTA
constexpr int kStages = 2;       // K/V ring depth
constexpr int kThreads = 384;         // three full warpgroups
constexpr int kMmaWarp = 8;
constexpr int kProducerWarp = 9;       // Q and K copies
constexpr int kVProducerWarp = 10;     // V copies (warp 11 only completes the third warpgroup)
// Register split: the kernel is launched with kLaunchRegs per thread (what
// __launch_bounds__(384, 1) allows); the two softmax warpgroups then grow to
// kSoftmaxRegs and the third warpgroup shrinks to kOtherRegs.  Both the CTA's
// pool (384 * 168 = 256 * 216 + 128 * 72) and each SM sub-partition's register
// file ((216 + 216 + 72) x 32 = 16128 <= 16384 per thread slot) are respected.
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 216;
constexpr int kOtherRegs = 72;
static_assert(kThreads * kLaunchRegs >= 256 * kSoftmaxRegs + 128 * kOtherRegs, "register split exceeds the pool");
static_assert((2 * kSoftmaxRegs + kOtherRegs) * 32 <= 16384, "register split exceeds a sub-partition");
constexpr uint32_t kTmemCols = 512;
constexpr int kSubBytes = 128 * 128;  // one [128 rows][64 bf16] swizzled sub-tile = 16 KB
constexpr int kPageRows = 16;         // tokens per page of a paged K/V pool
constexpr int kPageBytes = kPageRows * 128;  // one page's [16 rows][64 bf16] box: two 1 KB swizzle atoms
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kTau = 8.0f;          // rescale threshold, base-2 units

// Codes of the wait sites, recorded if a bounded wait gives up.
enum WaitSite : uint32_t {
    kSiteKEmpty = 1, kSiteVEmpty, kSiteQFull, kSiteKFull, kSitePFull, kSiteVFull, kSiteSFull, kSiteOFull,
    kSiteOFinal, kSiteQEmpty, kSiteOFree
};
template <int D, bool kFp8>
struct Layout {
    static constexpr int kElem = kFp8 ? 1 : 2;            // bytes per element of Q, K, V
    static constexpr int kSubCols = 128 / kElem;          // columns per 128-byte swizzled row
    static constexpr int kSubs = D / kSubCols;            // sub-tiles of kSubCols columns per row block
    static constexpr int kTileBytes = kSubs * kSubBytes;  // a [128][D] tile
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kTiles * kTileBytes;
    static constexpr int kOffV = kOffK + kStages * kTileBytes;
    static constexpr int kOffBar = kOffV + kStages * kTileBytes;
    static constexpr int kOffMask = kOffBar + 256;        // key-mask summaries, 8 bytes per batch row
    static constexpr int kBytes = kOffMask;
    __host__ __device__ static constexpr uint32_t colS(int i) { return (uint32_t)(i * 128); }
    __host__ __device__ static constexpr uint32_t colO(int i) { return (uint32_t)(256 + i * D); }
};

struct Bars {
    uint64_t q_full, q_empty;
    uint64_t k_full[kStages], k_empty[kStages];
    uint64_t v_full[kStages], v_empty[kStages];
    uint64_t s_full[kTiles], p_lo[kTiles], p_hi[kTiles], o_full[kTiles], o_free[kTiles];
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

// The MMA issue helpers put a whole tile's MMAs into one asm block.  Every
// shared-memory descriptor of a tile differs from the tile's first one only in
// the start-address field of its low word (16-byte units, no carry below 256 KB),
// and the high word (stride offset, version, 128-byte swizzle) is the same for
// the Q, K and V descriptors, so each MMA costs one or two 32-bit adds and the
// issuing warp, which shares its sub-partition with two busy softmax warps,
// needs few issue slots per MMA.  All lanes of the warp execute the block with
// the same operands; lane `leader` alone issues.
#define ATTN_QK_STEP(OFF)                                                        \
    "add.u32 al, %1, " #OFF ";\n\t"                                              \
    "add.u32 bl, %2, " #OFF ";\n\t"                                              \
    "mov.b64 da, {al, %3};\n\t"                                                  \
    "mov.b64 db, {bl, %3};\n\t"                                                  \
    "@e tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %4, t;\n\t"

__device__ __forceinline__ uint32_t desc_hi_sw128() { return (uint32_t)(smem_desc_sw128(0, 16, 1024) >> 32); }

// S = Q_i K_j^T: D/16 MMAs of K = 16, both operands K-major with 128-byte swizzle
// (k-steps of 32 bytes inside a 64-column sub-tile, sub-tiles 16 KB apart).
template <int D, bool kFp8>
__device__ __forceinline__ void issue_qk(bool leader, uint32_t d_tmem, uint32_t sq, uint32_t sk) {
    const uint32_t a_lo = (uint32_t)smem_desc_sw128(sq, 16, 1024);
    const uint32_t b_lo = (uint32_t)smem_desc_sw128(sk, 16, 1024);
    static_assert(D == 64 || D == 128, "head dim");
    if constexpr (kFp8) {
        // E4M3: K = 32 per MMA, i.e. 32 bytes of the single 128-byte swizzled row (D = 128)
        constexpr uint32_t idesc = idesc_e4m3_f32(BM, BN, 0, 0);
        const uint32_t hi = desc_hi_sw128();
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)
            asm volatile(
                "{\n\t.reg .pred e, p;\n\t.reg .b64 da, db;\n\t"
                "setp.ne.b32 e, %5, 0;\n\t"
                "setp.ne.b32 p, %6, 0;\n\t"
                "mov.b64 da, {%1, %3};\n\t"
                "mov.b64 db, {%2, %3};\n\t"
                "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], da, db, %4, p;\n\t}" ::"r"(d_tmem),
                "r"(a_lo + 2u * kk), "r"(b_lo + 2u * kk), "r"(hi), "r"(idesc), "r"((uint32_t)leader),
                "r"(kk > 0 ? 1u : 0u)
                : "memory");
    } else if constexpr (D == 128) {
        asm volatile(
            "{\n\t.reg .pred e, t, f;\n\t.reg .b32 al, bl;\n\t.reg .b64 da, db;\n\t"
            "setp.ne.b32 e, %5, 0;\n\t"
            "setp.eq.b32 t, %5, %5;\n\t"
            "setp.ne.b32 f, %5, %5;\n\t"
            "mov.b64 da, {%1, %3};\n\t"
            "mov.b64 db, {%2, %3};\n\t"
            "@e tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %4, f;\n\t"
            ATTN_QK_STEP(2) ATTN_QK_STEP(4) ATTN_QK_STEP(6)
            ATTN_QK_STEP(1024) ATTN_QK_STEP(1026) ATTN_QK_STEP(1028) ATTN_QK_STEP(1030)
            "}" ::"r"(d_tmem), "r"(a_lo), "r"(b_lo), "r"(desc_hi_sw128()), "r"(idesc_bf16_f32(BM, BN, 0, 0)),
            "r"((uint32_t)leader)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred e, t, f;\n\t.reg .b32 al, bl;\n\t.reg .b64 da, db;\n\t"
            "setp.ne.b32 e, %5, 0;\n\t"
            "setp.eq.b32 t, %5, %5;\n\t"
            "setp.ne.b32 f, %5, %5;\n\t"
            "mov.b64 da, {%1, %3};\n\t"
            "mov.b64 db, {%2, %3};\n\t"
            "@e tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %4, f;\n\t"
            ATTN_QK_STEP(2) ATTN_QK_STEP(4) ATTN_QK_STEP(6)
            "}" ::"r"(d_tmem), "r"(a_lo), "r"(b_lo), "r"(desc_hi_sw128()), "r"(idesc_bf16_f32(BM, BN, 0, 0)),
            "r"((uint32_t)leader)
            : "memory");
    }
}
#undef ATTN_QK_STEP

// O_i (+)= P_i V_j over half `half` of the block's keys (64 keys), P from TMEM, V
// MN-major from shared memory (128-byte swizzle, 8-row groups 1 KB apart).
//   bf16: 4 MMAs of K = 16 keys; P packs 2 keys per TMEM column (8 columns per step);
//         64-column groups of V 16 KB apart; a 16-key step is 2 KB = 128 units.
//   E4M3: 2 MMAs of K = 32 keys; P packs 4 keys per column (8 columns per step); the
//         128 columns of V are one 128-byte group; a 32-key step is 4 KB = 256 units.
template <int D, bool kFp8>
__device__ __forceinline__ void issue_pv_half(bool leader, uint32_t d_tmem, uint32_t p_tmem, uint32_t sv, int half,
                                              bool accumulate) {
    const uint32_t b_lo = (uint32_t)smem_desc_sw128(sv, kSubBytes, 1024);
    const uint32_t hi = desc_hi_sw128();
    if constexpr (kFp8) {
        constexpr uint32_t idesc = idesc_e4m3_f32(BM, D, 0, 1);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int kk = 2 * half + q;
            asm volatile(
                "{\n\t.reg .pred e, p;\n\t.reg .b64 db;\n\t"
                "setp.ne.b32 e, %5, 0;\n\t"
                "setp.ne.b32 p, %6, 0;\n\t"
                "mov.b64 db, {%2, %3};\n\t"
                "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], db, %4, p;\n\t}" ::"r"(d_tmem),
                "r"(p_tmem + kk * 8), "r"(b_lo + kk * 256), "r"(hi), "r"(idesc), "r"((uint32_t)leader),
                "r"((accumulate || q > 0) ? 1u : 0u)
                : "memory");
        }
    } else {
        constexpr uint32_t idesc = idesc_bf16_f32(BM, D, 0, 1);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int kk = 4 * half + q;
            asm volatile(
                "{\n\t.reg .pred e, p;\n\t.reg .b64 db;\n\t"
                "setp.ne.b32 e, %5, 0;\n\t"
                "setp.ne.b32 p, %6, 0;\n\t"
                "mov.b64 db, {%2, %3};\n\t"
                "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %4, p;\n\t}" ::"r"(d_tmem),
                "r"(p_tmem + kk * 8), "r"(b_lo + kk * 128), "r"(hi), "r"(idesc), "r"((uint32_t)leader),
                "r"((accumulate || q > 0) ? 1u : 0u)
                : "memory");
        }
    }
}

// Make the compiler treat registers filled by tcgen05.ld as defined only after
// tcgen05.wait::ld (this volatile statement is ordered after the wait).
__device__ __forceinline__ void pin8(uint32_t* r) {
    asm volatile("" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]));
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// O rows of this warp's TMEM lane quarter times alpha, 64 columns per TMEM round trip.
template <int D>
__device__ __forceinline__ void rescale_o_rows(uint32_t taddr, float alpha) {
    const uint64_t a2 = f2_make(alpha, alpha);
#pragma unroll 1
    for (int c = 0; c < D / 64; ++c) {
        uint32_t o[64];
        tmem_ld32(taddr + 64 * c, o);
        tmem_ld32(taddr + 64 * c + 32, o + 32);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 64; e += 8) pin8(o + e);
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
            float x0, x1;
            f2_split(f2_mul(f2_make(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), a2), x0, x1);
            o[e] = __float_as_uint(x0);
            o[e + 1] = __float_as_uint(x1);
        }
        tmem_st32(taddr + 64 * c, o);
        tmem_st32(taddr + 64 * c + 32, o + 32);
    }
}

// Work items: (pair of query tiles, head, batch), in one grid-wide order with
// the heaviest causal pairs first.  The persistent CTAs walk it in rounds of
// gridDim.x items, forwards in even rounds and backwards in odd ones, so every
// CTA gets a mix of heavy and light causal items.
__device__ __forceinline__ int item_of(int cta, int k, int grid) {
    return k * grid + ((k & 1) ? grid - 1 - cta : cta);
}

struct ItemGeom {
    int m0, h, b, g;       // first query row, head, batch row, kv head
    int nb[kTiles];        // key blocks each tile visits (0 for a tile past the last query row)
    int n_blk, q_tiles;    // key blocks of the item; tiles that hold query rows
    int first_unkept;      // smallest masked-out key of the batch row (n_kv if none)
    int n_kv, offset;      // keys of the batch row; causal: row i keeps keys j <= i + offset
};

template <int D, bool kPaged, bool kFp8>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_bf16_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                    const __grid_constant__ CUtensorMap tv, const FwdArgs a, unsigned int* status) {
    using L = Layout<D, kFp8>;
    static_assert(!kFp8 || (D == 128 && !kPaged), "FP8 inputs: head dim 128, contiguous keys");
    extern __shared__ uint8_t smem_raw[];
    // tiles need 1024-byte alignment for the 128-byte swizzle atoms
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    Bars& bar = *reinterpret_cast<Bars*>(smem + L::kOffBar);
    int* const mask_fu = reinterpret_cast<int*>(smem + L::kOffMask);  // [B] first excluded key
    int* const mask_lk = mask_fu + a.B;                                  // [B] last kept key

    const int tid = threadIdx.x;
    const int warp = tid / 32;
    const int n_pairs = (a.n_q + kTiles * BM - 1) / (kTiles * BM);
    const int n_items = n_pairs * a.H * a.B;
    const int grid = (int)gridDim.x, cta = (int)blockIdx.x;

    if (tid == 0) {
        mbar_init(&bar.q_full, 1);
        mbar_init(&bar.q_empty, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bar.k_full[s], 1);
            mbar_init(&bar.k_empty[s], 1);
            mbar_init(&bar.v_full[s], 1);
            mbar_init(&bar.v_empty[s], 1);
        }
        for (int i = 0; i < kTiles; ++i) {
            mbar_init(&bar.s_full[i], 1);
            mbar_init(&bar.p_lo[i], 128);
            mbar_init(&bar.p_hi[i], 128);
            mbar_init(&bar.o_full[i], 1);
            mbar_init(&bar.o_free[i], 128);
        }
        bar.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&bar.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (a.key_mask != nullptr) {
        // each batch row's key mask summarised once: first excluded and last kept key
        const int lane = tid % 32;
        for (int bb = warp; bb < a.B; bb += kThreads / 32) {
            const uint8_t* km = a.key_mask + (size_t)bb * a.n_kv;
            int fu = a.n_kv, lk = -1;
            if ((reinterpret_cast<uintptr_t>(km) & 15u) == 0 && (a.n_kv & 15) == 0) {
                // 16 mask bytes per lane and load
                for (int j16 = lane; j16 < a.n_kv / 16; j16 += 32) {
                    const uint4 w = reinterpret_cast<const uint4*>(km)[j16];
                    const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int t = 0; t < 16; ++t) {
                        const int j = j16 * 16 + t;
                        if ((wd[t / 4] >> (8 * (t % 4))) & 0xffu) lk = j;
                        else fu = min(fu, j);
                    }
                }
            } else {
                for (int j = lane; j < a.n_kv; j += 32) {
                    if (km[j]) lk = j;
                    else fu = min(fu, j);
                }
            }
#pragma unroll
            for (int sh = 16; sh > 0; sh >>= 1) {
                fu = min(fu, __shfl_xor_sync(0xffffffffu, fu, sh));
                lk = max(lk, __shfl_xor_sync(0xffffffffu, lk, sh));
            }
            if (lane == 0) {
                mask_fu[bb] = fu;
                mask_lk[bb] = lk;
            }
        }
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar.tmem_base;

    auto geometry = [&](int item) {
        ItemGeom gm;
        int pair;
        if constexpr (!kPaged) {
            // pairs outermost (heaviest causal pairs first), then heads and batch rows: one
            // round of items spans every kv head of a few pairs, whose K/V stay in L2
            const int hb = a.H * a.B;
            const int r = item / hb, rest = item % hb;
            pair = a.causal ? n_pairs - 1 - r : r;
            gm.h = rest % a.H;
            gm.b = rest / a.H;
        } else {
            // sequences' kv heads outermost, then the pairs of the query block (heaviest
            // first), then the query heads of the group: a round of items touches the
            // scattered pages of only a few (sequence, kv head) caches
            const int G = a.H / a.H_kv;
            const int hg = item % G, rest = item / G;
            const int pr = rest % n_pairs, bg = rest / n_pairs;
            pair = a.causal ? n_pairs - 1 - pr : pr;
            gm.b = bg / a.H_kv;
            gm.h = (bg % a.H_kv) * G + hg;
        }
        gm.g = gm.h / (a.H / a.H_kv);
        gm.m0 = pair * kTiles * BM;
        gm.n_kv = a.n_kv;
        if (kPaged) gm.n_kv = min(max(a.seq_lens[gm.b], 0), a.max_pages * kPageRows);
        gm.offset = gm.n_kv - a.n_q;
        const int last_kept = a.key_mask ? mask_lk[gm.b] : gm.n_kv - 1;
        gm.first_unkept = a.key_mask ? mask_fu[gm.b] : gm.n_kv;
#pragma unroll
        for (int i = 0; i < kTiles; ++i) {
            const int r0 = gm.m0 + i * BM;
            int kv_hi = min(gm.n_kv, last_kept + 1);
            if (a.causal) kv_hi = min(kv_hi, r0 + BM + gm.offset);
            gm.nb[i] = (r0 < a.n_q && kv_hi > 0) ? (kv_hi + BN - 1) / BN : 0;
        }
        gm.n_blk = max(gm.nb[0], gm.nb[1]);
        gm.q_tiles = (gm.m0 + BM < a.n_q) ? 2 : 1;
        return gm;
    };

    const uint32_t sQ = smem_u32(smem + L::kOffQ);
    const uint32_t sK = smem_u32(smem + L::kOffK);
    const uint32_t sV = smem_u32(smem + L::kOffV);

    if (warp >= 8) {
      // every warp of the third warpgroup runs the same register shrink, then its role
      regs_shrink<kOtherRegs>();
      if (warp == kProducerWarp || warp == kVProducerWarp) {
        // Two producer warps: warp 9 copies Q and K, warp 10 copies V, so a K copy waiting
        // for its ring slot never holds back the V copy the next P V needs.  Each whole warp
        // walks the item loop; lane 0 waits for ring slots and arms the barriers.  Contiguous
        // tiles are copied by lane 0; with paged keys lane p copies the block's p-th page, so
        // the eight page copies of a tile are issued at once.
        const bool do_k = warp == kProducerWarp, do_v = !do_k;
        const int lane = tid % 32;
        if (lane == 0) {
            tma_prefetch_desc(&tq);
            tma_prefetch_desc(&tk);
            tma_prefetch_desc(&tv);
        }
        volatile int* ab = &bar.abort_flag;
        auto wait0 = [&](uint64_t* b_, uint32_t parity, uint32_t site) {
            int r = 1;
            if (lane == 0) r = mbar_wait(b_, parity, ab, status, site) ? 1 : 0;
            return __shfl_sync(0xffffffffu, r, 0) != 0;
        };
        constexpr int kBlkPages = BN / kPageRows;
        // this lane's page id for key block j (lanes 0-7, paged keys): loaded a block ahead
        // of its copies; a page past the sequence's end stands in with one of its pages
        // (those rows are masked, and their V rows are zeroed before P V)
        auto fetch_page = [&](int j, const ItemGeom& gm) {
            if (!kPaged || lane >= kBlkPages) return 0;
            const int seq_pages = (gm.n_kv + kPageRows - 1) / kPageRows;  // >= 1: the block exists
            int page = a.block_table[(size_t)gm.b * a.max_pages + min(j * kBlkPages + lane, seq_pages - 1)];
            if (page < 0 || page >= a.num_pages) {
                atomicOr(status, ATTN_DEV_BAD_PAGE);
                page = 0;
            }
            return page;
        };
        // one key block's K or V tile: a 128-row box per 64 columns, or eight 16-row page boxes
        auto load_kv_tile = [&](uint8_t* dst, const CUtensorMap* map, uint64_t* full, int j, const ItemGeom& gm,
                                int page) {
            if constexpr (!kPaged) {
                // every query tile of the kv head reads these blocks again: L2 keeps them first
                if (lane == 0)
#pragma unroll
                    for (int s = 0; s < L::kSubs; ++s)
                        tma_load_4d_hint(dst + s * kSubBytes, map, full, s * L::kSubCols, j * BN, gm.g, gm.b,
                                         policy_evict_last());
            } else {
                if (lane < kBlkPages)
#pragma unroll
                    for (int s = 0; s < L::kSubs; ++s)
                        tma_load_4d(dst + s * kSubBytes + lane * kPageBytes, map, full, s * 64, gm.g, 0, page);
            }
        };
        uint32_t nq = 0, kc = 0, vc = 0;  // Q, K and V loads issued so far
        // test hook only: CTA 0 withholds its first V copy (and its transaction count), so the
        // MMA issuer's bounded wait for it runs out; nothing is issued that could land later
        bool drop_v = cta == 0 && (test_flags(status) & ATTN_TEST_DROP_FIRST_V) != 0;
        bool ok = true;
        for (int k = 0; ok; ++k) {
            const int item = item_of(cta, k, grid);
            if (item >= n_items) break;
            const ItemGeom gm = geometry(item);
            if (gm.n_blk == 0) continue;
            // the previous item's last S MMAs have read the Q tiles
            if (do_k && !wait0(&bar.q_empty, (nq & 1) ^ 1, kSiteQEmpty)) break;
            if (do_k && lane == 0) {
                mbar_arrive_expect_tx(&bar.q_full, gm.q_tiles * L::kTileBytes);
                // Q is read once: evict-first, so it does not push K and V out of L2
                for (int i = 0; i < gm.q_tiles; ++i)
#pragma unroll
                    for (int s = 0; s < L::kSubs; ++s)
                        tma_load_4d_hint(smem + L::kOffQ + i * L::kTileBytes + s * kSubBytes, &tq, &bar.q_full,
                                         s * L::kSubCols, gm.m0 + i * BM, gm.h, gm.b, policy_evict_first());
            }
            ++nq;
            int page = fetch_page(0, gm);
            for (int j = 0; j < gm.n_blk; ++j) {
                const int page_next = j + 1 < gm.n_blk ? fetch_page(j + 1, gm) : 0;
                if (do_k) {
                    const int st = kc % kStages;
                    if (!wait0(&bar.k_empty[st], ((kc / kStages) & 1) ^ 1, kSiteKEmpty)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) mbar_arrive_expect_tx(&bar.k_full[st], L::kTileBytes);
                    __syncwarp();
                    load_kv_tile(smem + L::kOffK + st * L::kTileBytes, &tk, &bar.k_full[st], j, gm, page);
                    ++kc;
                } else {
                    const int st = vc % kStages;
                    if (!wait0(&bar.v_empty[st], ((vc / kStages) & 1) ^ 1, kSiteVEmpty)) {
                        ok = false;
                        break;
                    }
                    if (!drop_v) {
                        if (lane == 0) mbar_arrive_expect_tx(&bar.v_full[st], L::kTileBytes);
                        __syncwarp();
                        load_kv_tile(smem + L::kOffV + st * L::kTileBytes, &tv, &bar.v_full[st], j, gm, page);
                    }
                    drop_v = false;
                    ++vc;
                }
                page = page_next;
            }
        }
        if (lane == 0 && bar.abort_flag) {
            // an aborted CTA must not exit with its bulk copies still landing in shared memory:
            // each producer waits (bounded) for the copies it issued
            if (do_k && nq > 0) mbar_drain(&bar.q_full, (nq - 1) & 1);
            for (uint32_t c = kc > kStages ? kc - kStages : 0; c < kc; ++c)
                mbar_drain(&bar.k_full[c % kStages], (c / kStages) & 1);
            for (uint32_t c = vc > kStages ? vc - kStages : 0; c < vc; ++c)
                mbar_drain(&bar.v_full[c % kStages], (c / kStages) & 1);
        }
      } else if (warp == kMmaWarp) {
        // The whole warp walks the issue loop with warp-uniform operands; lane 0
        // alone issues the MMAs and their commits.
        const bool leader = (tid % 32) == 0;
        volatile int* ab = &bar.abort_flag;
        uint32_t nq = 0, kc = 0, vc = 0;        // Q, K and V tiles consumed so far
        uint32_t tb[kTiles] = {0, 0};           // key blocks of each tile so far (S, P phases)
        uint32_t ni[kTiles] = {0, 0};           // items with blocks of each tile so far (O phases)
        bool ok = true;
        for (int k = 0; ok; ++k) {
            const int item = item_of(cta, k, grid);
            if (item >= n_items) break;
            const ItemGeom gm = geometry(item);
            if (gm.n_blk == 0) continue;
            ok = warp_wait(&bar.q_full, nq & 1, ab, status, kSiteQFull) &&
                 warp_wait(&bar.k_full[kc % kStages], (kc / kStages) & 1, ab, status, kSiteKFull);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int i = 0; i < kTiles; ++i)
                if (gm.nb[i] > 0) {
                    issue_qk<D, kFp8>(leader, tmem + L::colS(i), sQ + i * L::kTileBytes, sK + (kc % kStages) * L::kTileBytes);
                    mma_commit(leader, &bar.s_full[i]);
                }
            if (gm.n_blk == 1) mma_commit(leader, &bar.q_empty);  // the item's last S MMAs
            mma_commit(leader, &bar.k_empty[kc % kStages]);
            ++kc;
            for (int j = 0; ok && j < gm.n_blk; ++j) {
                const int sv = vc % kStages, sk = kc % kStages;
                const bool next = j + 1 < gm.n_blk;
                // V_j and K_{j+1} were requested a block ahead: wait for them here, off the
                // path from a tile's P to its P V and next S
                ok = warp_wait(&bar.v_full[sv], (vc / kStages) & 1, ab, status, kSiteVFull) &&
                     (!next || warp_wait(&bar.k_full[sk], (kc / kStages) & 1, ab, status, kSiteKFull));
                if (!ok) break;
                if (kPaged && (j + 1) * BN > gm.n_kv) {
                    // V rows past the sequence's end (the rest of its last page, stand-in pages)
                    // may hold anything, NaN included; their weights are 0, but 0 * NaN is not,
                    // so the warp zeroes those rows before the tensor core reads the tile
                    const int r_end = gm.n_kv - j * BN;
                    const uint32_t vb = sV + sv * L::kTileBytes;
                    for (int idx = tid % 32; idx < (BN - r_end) * (D / 8); idx += 32) {
                        const int r = r_end + idx / (D / 8), cc = idx % (D / 8);
                        st_shared_v4(vb + (cc / 8) * kSubBytes + r * 128 + (((cc % 8) ^ (r & 7)) << 4), 0u, 0u, 0u, 0u);
                    }
                    fence_proxy_async();
                    __syncwarp();
                }
#pragma unroll
                for (int i = 0; i < kTiles; ++i) {
                    if (j < gm.nb[i]) {
                        // the previous item's epilogue has read this tile's O
                        if (j == 0 && ni[i] > 0 &&
                            !warp_wait(&bar.o_free[i], (ni[i] - 1) & 1, ab, status, kSiteOFree)) {
                            ok = false;
                            break;
                        }
                        // the first half of P V starts while the softmax still exponentiates the
                        // second half of the row
                        if (!warp_wait(&bar.p_lo[i], tb[i] & 1, ab, status, kSitePFull)) { ok = false; break; }
                        tc_fence_after();
                        issue_pv_half<D, kFp8>(leader, tmem + L::colO(i), tmem + L::colS(i), sV + sv * L::kTileBytes, 0,
                                         j > 0);
                        if (!warp_wait(&bar.p_hi[i], tb[i] & 1, ab, status, kSitePFull)) { ok = false; break; }
                        tc_fence_after();
                        issue_pv_half<D, kFp8>(leader, tmem + L::colO(i), tmem + L::colS(i), sV + sv * L::kTileBytes, 1,
                                         true);
                        // only the epilogue waits for O (S_{j+1}'s completion already orders
                        // P_j V_j before the next block's rescale)
                        if (j == gm.nb[i] - 1) mma_commit(leader, &bar.o_full[i]);
                        ++tb[i];
                    }
                    if (i == kTiles - 1) mma_commit(leader, &bar.v_empty[sv]);
                    if (next && j + 1 < gm.nb[i]) {
                        issue_qk<D, kFp8>(leader, tmem + L::colS(i), sQ + i * L::kTileBytes, sK + sk * L::kTileBytes);
                        mma_commit(leader, &bar.s_full[i]);
                    }
                    if (next && i == kTiles - 1) {
                        if (j + 2 == gm.n_blk) mma_commit(leader, &bar.q_empty);  // the item's last S MMAs
                        mma_commit(leader, &bar.k_empty[sk]);
                    }
                }
                ++vc;
                if (next) ++kc;
            }
#pragma unroll
            for (int i = 0; i < kTiles; ++i) ni[i] += gm.nb[i] > 0 ? 1u : 0u;
            ++nq;
        }
      }
    } else {
        // ------------------------------------------------ softmax warpgroups (warps 0-7)
        regs_grow<kSoftmaxRegs>();
        const int ti = warp / 4;             // this warpgroup's query tile
        const int r = tid % 128;             // row within the tile = TMEM lane
        const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
        const uint32_t scol = L::colS(ti), ocol = L::colO(ti);
        const float sl2 = a.scale * kLog2e;
        // FP8: P is rounded to E4M3 (largest finite 448, smallest subnormal 2^-9), so the
        // reference follows every new maximum and P is measured 2^8 above it: weights stay
        // <= 256 and keep their bits down to 2^-17 of the row's maximum weight
        constexpr float kTauP = kFp8 ? 0.f : kTau;
        constexpr float kShift = kFp8 ? 8.f : 0.f;
        const int lane = tid % 32;
        uint32_t tb = 0, ni = 0;  // key blocks and items with blocks of this tile so far
        bool ok = true;
        for (int k = 0; ok; ++k) {
            const int item = item_of(cta, k, grid);
            if (item >= n_items) break;
            const ItemGeom gm = geometry(item);
            const int m0 = gm.m0, b = gm.b, h = gm.h;
            const int first_unkept = gm.first_unkept;
            const int row = m0 + ti * BM + r;
            const int n_kv = gm.n_kv, offset = gm.offset;
            const int row_limit = a.causal ? row + offset : 0x7fffffff;
            const int nbt = gm.nb[ti];
            float m_ref = -INFINITY;  // reference of u and l, base-2 units of the scaled score
            float l_run = 0.f;  // sum of the weights (log-sum-exp)
            float l_bf = 0.f;   // sum of the bf16-rounded weights (normalises O)
            // FP8 block scales: the scores of key block j are scale * s_Q * s_K[j] * (q8 . k8), and
            // V block j stands for s_V[j] * v8.  The factor s_V[j] / c_v (c_v the largest V descale of
            // the kv head, so the factor is <= 1) is added to the weights' exponent before they are
            // rounded to E4M3, and divided back out of both row sums, so O = c_v * (P V) / l.
            float c_q = sl2, c_v = 1.f;
            const float* k_desc = nullptr;
            const float* v_desc = nullptr;
            if constexpr (kFp8) {
                if (nbt > 0) {
                    const int nqb = (a.n_q + BM - 1) / BM, nkb = (n_kv + BN - 1) / BN;
                    const float sq = __ldg(a.q_descale + (size_t)(b * a.H + h) * nqb + (m0 / BM + ti));
                    k_desc = a.k_descale + (size_t)(b * a.H_kv + gm.g) * nkb;
                    v_desc = a.v_descale + (size_t)(b * a.H_kv + gm.g) * nkb;
                    float mxv = 0.f;
                    bool bad = !(sq > 0.f && sq < INFINITY);
                    for (int jj = lane; jj < nkb; jj += 32) {
                        const float sv = __ldg(v_desc + jj);
                        bad |= !(sv > 0.f && sv < INFINITY);
                        mxv = fmaxf(mxv, sv);
                    }
#pragma unroll
                    for (int sh = 16; sh > 0; sh >>= 1) mxv = fmaxf(mxv, __shfl_xor_sync(0xffffffffu, mxv, sh));
                    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(status, ATTN_DEV_BAD_SCALE);
                    c_q = sl2 * sq;
                    c_v = mxv;
                }
            }

            for (int j = 0; j < nbt; ++j, ++tb) {
                // this key block's score factor, and (FP8) its V factor's log2 and inverse
                float sl2j = sl2, lvj = 0.f, inv_r = 1.f;
                if constexpr (kFp8) {
                    const float sk = __ldg(k_desc + j), sv = __ldg(v_desc + j);
                    if (!(sk > 0.f && sk < INFINITY) && lane == 0) atomicOr(status, ATTN_DEV_BAD_SCALE);
                    sl2j = c_q * sk;
                    inv_r = c_v / sv;
                    lvj = -__log2f(inv_r);
                }
                if (!warp_wait(&bar.s_full[ti], tb & 1, &bar.abort_flag, status, kSiteSFull)) { ok = false; break; }
                tc_fence_after();
                const int n0 = j * BN;
                const bool need_mask = (n0 + BN > n_kv) ||
                                       (a.causal && n0 + BN - 1 > m0 + ti * BM + offset) ||
                                       (a.key_mask != nullptr && n0 + BN > first_unkept);
                // the score row from TMEM: columns 64-127 load while the maximum of 0-63 is taken
                uint32_t sraw[BN];
                tmem_ld32(tmem + lane_base + scol + 0, sraw + 0);
                tmem_ld32(tmem + lane_base + scol + 32, sraw + 32);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 64; c += 8) pin8(sraw + c);
                tmem_ld32(tmem + lane_base + scol + 64, sraw + 64);
                tmem_ld32(tmem + lane_base + scol + 96, sraw + 96);
                // excluded keys of 32-column group q set to -inf: a contiguous range (causal limit,
                // end of the keys) intersected with the batch row's key mask; the mask is the same
                // for every row, so each warp turns 32 of its bytes into a bit set with one ballot
                auto mask_group = [&](int q) {
                    const uint8_t* km = a.key_mask ? a.key_mask + (size_t)b * a.n_kv : nullptr;
                    const int rel = min(n_kv - 1, row_limit) - n0 - 32 * q;
                    uint32_t bits = rel >= 31 ? 0xffffffffu : (rel < 0 ? 0u : (0xffffffffu >> (31 - rel)));
                    if (km != nullptr) {
                        const int key = n0 + 32 * q + (tid % 32);
                        bits &= __ballot_sync(0xffffffffu, key < n_kv && km[key] != 0);
                    }
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        if (!((bits >> c) & 1u)) sraw[32 * q + c] = 0xff800000u;  // -inf
                };
                if (need_mask) {
                    mask_group(0);
                    mask_group(1);
                }
                // row maximum (three-input max, four independent chains)
                float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
                for (int c = 0; c < 64; c += 8) {
                    mx0 = max3f(mx0, __uint_as_float(sraw[c]), __uint_as_float(sraw[c + 1]));
                    mx1 = max3f(mx1, __uint_as_float(sraw[c + 2]), __uint_as_float(sraw[c + 3]));
                    mx2 = max3f(mx2, __uint_as_float(sraw[c + 4]), __uint_as_float(sraw[c + 5]));
                    mx3 = max3f(mx3, __uint_as_float(sraw[c + 6]), __uint_as_float(sraw[c + 7]));
                }
                tmem_wait_ld();
#pragma unroll
                for (int c = 64; c < 128; c += 8) pin8(sraw + c);
                if (need_mask) {
                    mask_group(2);
                    mask_group(3);
                }
#pragma unroll
                for (int c = 64; c < 128; c += 8) {
                    mx0 = max3f(mx0, __uint_as_float(sraw[c]), __uint_as_float(sraw[c + 1]));
                    mx1 = max3f(mx1, __uint_as_float(sraw[c + 2]), __uint_as_float(sraw[c + 3]));
                    mx2 = max3f(mx2, __uint_as_float(sraw[c + 4]), __uint_as_float(sraw[c + 5]));
                    mx3 = max3f(mx3, __uint_as_float(sraw[c + 6]), __uint_as_float(sraw[c + 7]));
                }
                const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2j;
                // move the reference only when the maximum passes it by more than kTau
                const bool move = mx > m_ref + kTauP;
                const float new_ref = move ? mx : m_ref;
                const float base = (new_ref == -INFINITY) ? 0.f : new_ref;
                const float alpha = move ? ex2_approx(m_ref - base) : 1.f;
                // S_j's completion implies P_{j-1} V_{j-1} completed: O is quiescent and may be rescaled
                // (FP8: after the first half of the weights, below)
                const bool resc = j > 0 && __any_sync(0xffffffffu, move);
                if (!kFp8 && resc) {
#pragma unroll 1
                    for (int c = 0; c < D / 16; ++c) {
                        uint32_t o[16];
                        tmem_ld16(tmem + lane_base + ocol + 16 * c, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st16(tmem + lane_base + ocol + 16 * c, o);
                    }
                }
                // P = 2^(S * scale * log2 e - base) packed to bf16 pairs, with the exact and the
                // rounded-weight row sums; each half of the row (64 keys = 32 packed columns) is
                // stored over the score columns already read and announced on its own barrier
                const uint64_t sl2x2 = f2_make(sl2j, sl2j);
                const uint64_t nbase2 = f2_make(kShift - base + lvj, kShift - base + lvj);
                uint64_t sum_e = f2_make(0.f, 0.f);
                float sr0 = 0.f, sr1 = 0.f;  // sums of the rounded weights (two chains)
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    if constexpr (!kFp8) {
                        uint32_t preg[32];
#pragma unroll
                        for (int c = 0; c < 64; c += 2) {
                            const int k = 64 * half + c;
                            const uint64_t x2 = f2_fma(f2_make(__uint_as_float(sraw[k]), __uint_as_float(sraw[k + 1])),
                                                       sl2x2, nbase2);
                            float x0, x1;
                            f2_split(x2, x0, x1);
                            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                            const uint32_t pk = pack_bf16x2(p0, p1);
                            preg[c / 2] = pk;
                            sum_e = f2_add(sum_e, f2_make(p0, p1));
                            // the two bf16 weights added into fp32 as they are (mixed-precision adds)
                            asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
                                "add.rn.f32.bf16 %0, lo, %0;\n\tadd.rn.f32.bf16 %1, hi, %1;\n\t}"
                                : "+f"(sr0), "+f"(sr1) : "r"(pk));
                        }
                        tmem_st32(tmem + lane_base + scol + 32 * half, preg);
                    } else {
                        // four E4M3 weights per TMEM column: 64 keys = 16 columns per half
                        uint32_t preg[16];
#pragma unroll
                        for (int c = 0; c < 64; c += 4) {
                            const int k = 64 * half + c;
                            const uint64_t xa = f2_fma(f2_make(__uint_as_float(sraw[k]), __uint_as_float(sraw[k + 1])),
                                                       sl2x2, nbase2);
                            const uint64_t xb = f2_fma(f2_make(__uint_as_float(sraw[k + 2]),
                                                               __uint_as_float(sraw[k + 3])),
                                                       sl2x2, nbase2);
                            float x0, x1, x2, x3;
                            f2_split(xa, x0, x1);
                            f2_split(xb, x2, x3);
                            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                            const float p2 = ex2_approx(x2), p3 = ex2_approx(x3);
                            const uint32_t w = pack_e4m3x4(p0, p1, p2, p3);
                            preg[c / 4] = w;
                            sum_e = f2_add(sum_e, f2_add(f2_make(p0, p1), f2_make(p2, p3)));
                            // the four rounded weights widened exactly to f16, added pairwise in f16x2
                            // (two E4M3 values add with error 2^-11 relative at most), then into fp32
                            asm("{\n\t.reg .b16 lo, hi, s0, s1;\n\t.reg .b32 f01, f23, s;\n\t"
                                "mov.b32 {lo, hi}, %2;\n\t"
                                "cvt.rn.f16x2.e4m3x2 f01, lo;\n\t"
                                "cvt.rn.f16x2.e4m3x2 f23, hi;\n\t"
                                "add.rn.f16x2 s, f01, f23;\n\t"
                                "mov.b32 {s0, s1}, s;\n\t"
                                "add.rn.f32.f16 %0, s0, %0;\n\t"
                                "add.rn.f32.f16 %1, s1, %1;\n\t}"
                                : "+f"(sr0), "+f"(sr1) : "r"(w));
                        }
                        tmem_st16(tmem + lane_base + scol + 16 * half, preg);
                        // FP8 moves the reference at every new maximum, so most blocks rescale O:
                        // here, where half of the score registers are free, 64 columns per TMEM
                        // round trip, before the first half of P is announced
                        if (half == 0 && resc) rescale_o_rows<D>(tmem + lane_base + ocol, alpha);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(half == 0 ? &bar.p_lo[ti] : &bar.p_hi[ti]);
                }
                float e0, e1;
                f2_split(sum_e, e0, e1);
                l_run = l_run * alpha + (e0 + e1) * inv_r;
                l_bf = l_bf * alpha + (sr0 + sr1) * inv_r;
                m_ref = new_ref;
            }

            // epilogue: O / l in bf16 (or fp32) and the log-sum-exp (natural log of the scaled scores)
            if (ok && nbt > 0) {
                ok = warp_wait(&bar.o_full[ti], ni & 1, &bar.abort_flag, status, kSiteOFinal);
                tc_fence_after();
            }
            const bool has = ok && nbt > 0 && l_run > 0.f && l_bf > 0.f;
            const float inv = has ? (kFp8 ? c_v / l_bf : 1.f / l_bf) : 0.f;
            const size_t orow_off = ((size_t)(b * a.H + h) * a.n_q + row) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                if (ok && nbt > 0) {
                    tmem_ld32(tmem + lane_base + ocol + 32 * c, o);
                    tmem_wait_ld();
                }
                if (row < a.n_q) {
                    if (a.o_f32) {
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<float*>(a.o) + orow_off + 32 * c);
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = has ? __float_as_uint(__uint_as_float(o[e]) * inv) : 0u;
#pragma unroll
                        for (int e = 0; e < 8; ++e) dst[e] = make_uint4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
                    } else {
                        uint32_t w[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            w[e] = has ? pack_bf16x2(__uint_as_float(o[2 * e]) * inv,
                                                     __uint_as_float(o[2 * e + 1]) * inv)
                                       : 0u;
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) + orow_off + 32 * c);
                        // O is written once: evict-first, like Q
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            asm volatile("st.global.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(dst + e),
                                         "r"(w[4 * e]), "r"(w[4 * e + 1]), "r"(w[4 * e + 2]), "r"(w[4 * e + 3]),
                                         "l"(policy_evict_first()) : "memory");
                    }
                }
            }
            if (a.lse != nullptr && row < a.n_q)
                a.lse[(size_t)(b * a.H + h) * a.n_q + row] =
                    has ? (m_ref + log2f(l_run) - kShift) * 0.6931471805599453f : -INFINITY;
            if (nbt > 0) {
                // this tile's O columns may take the next item's P V
                tc_fence_before();
                mbar_arrive(&bar.o_free[ti]);
                ++ni;
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

template <int D, bool kPaged, bool kFp8>
cudaError_t launch_d(const FwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     unsigned int* status, cudaStream_t stream) {
    // at least ~116 KB so that one CTA (and one 512-column TMEM allocation) sits on each SM
    constexpr int kMinSmem = 118 * 1024;
    const int smem = std::max(Layout<D, kFp8>::kBytes + 1024 + (a.key_mask ? 8 * a.B : 0), kMinSmem);
    static std::atomic<unsigned long long> ready{0};
    static std::atomic<int> sm_count[64];
    int dev = 0;
    cudaError_t e = setup_once_per_device(ready, &dev, [](int device) {
        auto kern = fwd_bf16_kernel<D, kPaged, kFp8>;
        // the largest request this launcher makes fits under the device's opt-in maximum
        int optin = 0;
        cudaError_t r = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
        if (r == cudaSuccess) r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
        if (r != cudaSuccess) return r;
        // the in-kernel register split assumes exactly kLaunchRegs per thread at launch
        cudaFuncAttributes fa;
        r = cudaFuncGetAttributes(&fa, kern);
        if (r != cudaSuccess) return r;
        if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
        // each CTA allocates all 512 TMEM columns, so exactly one may be resident per SM (at the
        // smallest request; larger ones leave still less room)
        int per_sm = 0;
        r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, kMinSmem);
        if (r != cudaSuccess) return r;
        if (per_sm != 1) return cudaErrorInvalidConfiguration;
        int sms = 0;
        r = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
        if (r == cudaSuccess && device < 64) sm_count[device].store(sms, std::memory_order_relaxed);
        return r;
    });
    if (e != cudaSuccess) return e;
    int sms = dev < 64 ? sm_count[dev].load(std::memory_order_relaxed) : 0;
    if (sms <= 0) {
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
    }
    // persistent: one CTA per SM, each walking its share of the work items
    const long long n_items = (long long)((a.n_q + kTiles * BM - 1) / (kTiles * BM)) * a.H * a.B;
    const int grid = (int)std::min<long long>(sms, n_items);
    fwd_bf16_kernel<D, kPaged, kFp8><<<grid, kThreads, smem, stream>>>(tq, tk, tv, a, status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_bf16_sm100(const FwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                                  const CUtensorMap& tv, unsigned int* status, cudaStream_t stream) {
    switch (a.d) {
        case 64:
            if (a.fp8) return cudaErrorInvalidValue;
            return a.block_table ? launch_d<64, true, false>(a, tq, tk, tv, status, stream)
                                 : launch_d<64, false, false>(a, tq, tk, tv, status, stream);
        case 128:
            if (a.fp8) return a.block_table ? cudaErrorInvalidValue : launch_d<128, false, true>(a, tq, tk, tv, status, stream);
            return a.block_table ? launch_d<128, true, false>(a, tq, tk, tv, status, stream)
                                 : launch_d<128, false, false>(a, tq, tk, tv, status, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace attn
