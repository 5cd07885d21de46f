// Internal declarations shared by the library's translation units (not part of the C ABI).
#pragma once
#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/attn_testing.h"  // test flags (status block word 6)

// Bits of the device status word (read and cleared by attn_check_status).
#define ATTN_DEV_TIMEOUT 0x1u     // a bounded wait gave up
#define ATTN_DEV_BAD_PAGE 0x2u    // a block-table entry outside [0, num_pages)
#define ATTN_DEV_BAD_LEN 0x4u     // a sequence length outside [0, max_seq_len]
#define ATTN_DEV_BAD_SCALE 0x8u   // an FP8 block descale that is not finite and > 0
#define ATTN_DEV_SMEM_LAYOUT 0x10u  // the dynamic shared memory cannot hold a kernel's aligned layout

namespace attn {

// One-time per-device setup before a kernel's launches on that device (function attributes,
// device queries).  Each call site owns one mask: bit i is set once `setup(i)` succeeded on
// device i (devices 0-63; others run it on every call).  Writes the current device to *dev.
// Like the other per-device caches of this library, it does not survive cudaDeviceReset.
template <typename F>
cudaError_t setup_once_per_device(std::atomic<unsigned long long>& mask, int* dev, F&& setup) {
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return e;
    const bool cached = *dev >= 0 && *dev < 64;
    if (cached && ((mask.load(std::memory_order_acquire) >> *dev) & 1ull)) return cudaSuccess;
    e = setup(*dev);
    if (e == cudaSuccess && cached) mask.fetch_or(1ull << *dev, std::memory_order_acq_rel);
    return e;
}

// Forward problem, row-major contiguous: q/o [B, H, n_q, d], k/v [B, H_kv, n_kv, d],
// lse [B, H, n_q] fp32 (may be null), key_mask [B, n_kv] uint8 (may be null).
struct FwdArgs {
    const void* q;
    const void* k;
    const void* v;
    void* o;
    float* lse;
    const uint8_t* key_mask;
    int B, H, H_kv, n_q, n_kv, d;
    float scale;
    int causal;
    int o_f32;            // bf16 inputs: write O as fp32 instead of bf16
    // paged keys and values (null block_table: contiguous K and V): k and v are the
    // page pools [num_pages, 16, H_kv, d]; batch row b is a sequence of seq_lens[b]
    // tokens whose last n_q positions are the query rows
    const int32_t* block_table;  // [B, max_pages]
    const int32_t* seq_lens;     // [B]
    int max_pages, num_pages;
    // FP8 E4M3 inputs (fp8 = 1): q, k and v hold E4M3 bytes; every element's value is its
    // decoded value times its block's descale, one per 128 rows of each head:
    // q_descale [B, H, ceil(n_q / 128)], k_descale and v_descale [B, H_kv, ceil(n_kv / 128)]
    int fp8;
    const float* q_descale;
    const float* k_descale;
    const float* v_descale;
};

struct DecodeArgs {
    const void* q;          // [S, H, d] bf16
    const void* k_pages;    // [P, page, H_kv, d] bf16
    const void* v_pages;
    const int32_t* block_table;  // [S, max_pages]
    const int32_t* seq_lens;     // [S]
    int num_seqs, H, H_kv, d, page_size, max_pages, num_pages, max_seq_len, split_tokens, n_splits;
    float scale;
    float* part_ml;   // [S, H, n_splits, 4]: m (base 2), l for the LSE, l that normalises u, unused
    float* part_u;    // [S, H, n_splits, d]
    void* o;          // [S, H, d] bf16
    float* lse;       // [S, H] or null
};

// Backward problem (bf16, row-major contiguous): q/o/d_o/dq [B, H, n_q, d], k/v/dk/dv
// [B, H_kv, n_kv, d], lse [B, H, n_q] fp32 (natural log, as the forward writes it),
// key_mask [B, n_kv] uint8 or null.  ws_l2 / ws_dd: workspace [B * H][n_q_pad] fp32
// (n_q_pad = n_q rounded up to 128) for LSE * log2(e) and dO . O per query row.
struct BwdArgs {
    const void* q;
    const void* k;
    const void* v;
    const void* o;
    const void* d_o;
    const float* lse;
    void* dq;
    void* dk;
    void* dv;
    const uint8_t* key_mask;
    int B, H, H_kv, n_q, n_kv, d, n_q_pad;
    float scale;
    int causal;
    float* ws_l2;
    float* ws_dd;
};

// Address of this device's status block (host side): [0] flag bits, [1..3]
// where the first bounded wait gave up (site | warp << 8, block, parity), [4..5]
// the test wait limit in ns (0 = the default), [6] test flags, [7] unused.
unsigned int* device_status_word();
void set_last_error(const char* msg);  // the text attn_last_error() returns on this host thread

cudaError_t launch_fwd_f32(const FwdArgs& a, unsigned int* status, cudaStream_t stream);
cudaError_t launch_fwd_bf16_sm100(const FwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                                  const CUtensorMap& tv, unsigned int* status, cudaStream_t stream);
cudaError_t launch_decode(const DecodeArgs& a, unsigned int* status, cudaStream_t stream);
cudaError_t launch_decode_mma(const DecodeArgs& a, const CUtensorMap& tk, const CUtensorMap& tv,
                              unsigned int* status, cudaStream_t stream);
cudaError_t launch_decode_merge(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_bwd(const BwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, unsigned int* status, cudaStream_t stream);

}  // namespace attn
