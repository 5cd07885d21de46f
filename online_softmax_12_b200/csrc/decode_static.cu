// attn_decode_paged_static: paged decode for callers that cannot allocate
// device memory.
//
// Some callers have no way to hand the library a workspace: code that runs
// where cudaMalloc is forbidden or unavailable (inside a host callback or a
// custom allocator's own path, under a memory budget that must not move, or
// in a plugin whose host framework owns every allocation).  For them this
// entry point keeps the split-KV partial states in a file-scope device array
// of fixed size instead of a caller-provided workspace, and otherwise runs
// exactly the kernels of attn_decode_paged.
//
// The array is a host-side stand-in in host code: its address on the device
// is looked up once per device with cudaGetSymbolAddress and that device
// pointer is what the kernels receive.  The address is cached for the life of
// the process: after cudaDeviceReset the module may load elsewhere, so the
// library must not be called again on a device that was reset.
#include <cstdio>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/attn.h"
#include "internal.h"

namespace {

// 32 MiB: enough for 64 sequences x 32 heads x 16 splits of partial states of
// 4 + d fp32 each (m, the two normalisers and a pad, then u: 132 floats at
// d = 128), about 17.3 MB; every GPU that loads the library holds it.
constexpr size_t kScratchBytes = 32ull << 20;
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_dev[kMaxDevices] = {};

// Device address of this device's scratch array, looked up on first use with
// that device current.  Returns nullptr (and records why) on failure.
void* scratch_for_current_device() {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        char msg[160];
        snprintf(msg, sizeof msg, "attn_decode_paged_static: cudaGetDevice: %s", cudaGetErrorString(e));
        attn::set_last_error(msg);
        return nullptr;
    }
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (g_scratch_dev[dev] == nullptr) {
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
        if (e != cudaSuccess || ptr == nullptr) {
            char msg[160];
            snprintf(msg, sizeof msg, "attn_decode_paged_static: cudaGetSymbolAddress(scratch): %s",
                     cudaGetErrorString(e));
            attn::set_last_error(msg);
            return nullptr;
        }
        g_scratch_dev[dev] = ptr;
    }
    return g_scratch_dev[dev];
}

}  // namespace

extern "C" {

attn_status_t attn_decode_paged_static(const void* q, const void* k_pages, const void* v_pages,
                                       const int32_t* block_table, const int32_t* seq_lens, int num_seqs, int H,
                                       int H_kv, int d, int page_size, int max_pages_per_seq, int num_pages,
                                       int max_seq_len, int split_tokens, float scale, void* o, float* lse,
                                       void* stream) {
    const size_t need = attn_decode_workspace_bytes(num_seqs, H, H_kv, d, max_seq_len, split_tokens);
    if (need == 0) {
        // invalid sizes: let the regular entry point produce its precise message
        return attn_decode_paged(q, k_pages, v_pages, block_table, seq_lens, num_seqs, H, H_kv, d, page_size,
                                 max_pages_per_seq, num_pages, max_seq_len, split_tokens, scale, nullptr, 0, o,
                                 lse, stream);
    }
    if (need > kScratchBytes) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "attn_decode_paged_static: these sizes need %zu bytes of partial states, more than the fixed "
                 "%zu-byte scratch; use attn_decode_paged with a workspace, or larger split_tokens",
                 need, kScratchBytes);
        attn::set_last_error(msg);
        return ATTN_ERR_INVALID_ARG;
    }
    void* scratch = scratch_for_current_device();
    if (scratch == nullptr) return ATTN_ERR_CUDA;
    return attn_decode_paged(q, k_pages, v_pages, block_table, seq_lens, num_seqs, H, H_kv, d, page_size,
                             max_pages_per_seq, num_pages, max_seq_len, split_tokens, scale, scratch, kScratchBytes,
                             o, lse, stream);
}

}  // extern "C"
