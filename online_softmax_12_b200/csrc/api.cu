// C ABI of libattn.so: argument validation, TMA descriptor encoding, dispatch,
// and the per-device status word.  Every entry point validates all host-side
// arguments before launching anything.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>
#include <string>

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "../../include/attn.h"
#include "../../include/attn_testing.h"
#include "internal.h"
#include "ptx.cuh"

namespace attn {
namespace {

// The per-device status block: words 0-3 are read and cleared by attn_check_status,
// words 4-6 hold the test hook's wait limit and flags (zero in normal use).
__device__ __align__(16) unsigned int g_status_word[8];

thread_local std::string t_last_error;

attn_status_t fail(attn_status_t st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
attn_status_t fail(attn_status_t st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    t_last_error = buf;
    return st;
}

attn_status_t cuda_fail(cudaError_t e, const char* where) {
    return fail(ATTN_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr int kMaxDevices = 64;
std::mutex g_mu;
std::atomic<unsigned int*> g_status_addr[kMaxDevices] = {};
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_encode == nullptr) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    return g_encode;
}

// 4-D bf16 tensor [outer][heads][rows][d] seen by TMA as (d, rows, heads, outer),
// boxes of 64 columns x box_rows rows, 128-byte swizzle, zero fill out of bounds.
bool encode_rows_map(CUtensorMap* map, const void* base, int d, int rows, int heads, int outer, int box_rows) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)heads, (cuuint64_t)outer};
    cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)rows * d * 2, (cuuint64_t)heads * rows * d * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)box_rows, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The same for one-byte elements (FP8 E4M3): boxes of 128 columns (one 128-byte swizzled row).
bool encode_rows_map_u8(CUtensorMap* map, const void* base, int d, int rows, int heads, int outer, int box_rows) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)heads, (cuuint64_t)outer};
    cuuint64_t strides[3] = {(cuuint64_t)d, (cuuint64_t)rows * d, (cuuint64_t)heads * rows * d};
    cuuint32_t box[4] = {128, (cuuint32_t)box_rows, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Paged pool [pages][page_size][H_kv][d] bf16 seen by TMA as (d, H_kv, page_size, pages),
// boxes of 64 columns x 1 head x page_size slots (one page's rows of one kv head), 128-byte swizzle.
bool encode_pages_map(CUtensorMap* map, const void* base, int d, int H_kv, int page_size, int num_pages) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H_kv, (cuuint64_t)page_size, (cuuint64_t)num_pages};
    cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H_kv * d * 2, (cuuint64_t)page_size * H_kv * d * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)page_size, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

__global__ void fill_empty_rows(void* o, float* lse, size_t n_rows, int d, int elem_bytes) {
    const size_t n_words = n_rows * (size_t)d * elem_bytes / 4;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n_words; i += (size_t)gridDim.x * blockDim.x)
        static_cast<uint32_t*>(o)[i] = 0u;
    if (lse != nullptr)
        for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n_rows; i += (size_t)gridDim.x * blockDim.x)
            lse[i] = -INFINITY;
}

// Tokens per split: as many as possible (fewer partial states, less per-CTA
// start-up) while leaving about 2048 CTAs (at three per SM, several waves) for
// a batch at max_seq_len; a multiple of 16 in [16, 1024].
int choose_split(int num_seqs, int H_kv, int max_seq_len) {
    int t = 1024;
    while (t > 16 && (long long)num_seqs * H_kv * ((max_seq_len + t - 1) / t) < 2048) t /= 2;
    return t;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct DecodeLayout {
    int split_tokens, n_splits;
    size_t off_u, bytes;
};

// Splits per sequence of the single-launch decode (the cluster size): 2, or 1 for a
// single page (clusters of 2 measured fastest: a cluster starts only when all its CTAs
// fit at once, and its CTAs wait for the slowest at the merge barrier).
int one_launch_splits(int max_seq_len) {
    const int pages = (max_seq_len + 15) / 16;
    int c = 2;
    while (c > 1 && c > pages) c /= 2;
    return c;
}

bool decode_layout(int num_seqs, int H, int H_kv, int d, int max_seq_len, int split_tokens, DecodeLayout* out) {
    if (num_seqs < 0 || H <= 0 || H_kv <= 0 || d <= 0 || max_seq_len < 0 || split_tokens < ATTN_DECODE_ONE_LAUNCH)
        return false;
    if (split_tokens == ATTN_DECODE_ONE_LAUNCH) {
        // no partial state leaves the chip: no workspace
        out->split_tokens = 0;
        out->n_splits = -one_launch_splits(max_seq_len);
        out->off_u = 0;
        out->bytes = 16;
        return true;
    }
    const int t = split_tokens > 0 ? split_tokens : choose_split(num_seqs, H_kv, max_seq_len);
    const int n_splits = max_seq_len > 0 ? (max_seq_len + t - 1) / t : 1;
    const size_t slots = (size_t)num_seqs * H * n_splits;
    out->split_tokens = t;
    out->n_splits = n_splits;
    out->off_u = align_up(slots * 4 * sizeof(float), 256);
    out->bytes = out->off_u + align_up(slots * (size_t)d * sizeof(float), 256);
    if (out->bytes == 0) out->bytes = 256;
    return true;
}

}  // namespace

unsigned int* device_status_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    unsigned int* cached = g_status_addr[dev].load(std::memory_order_acquire);
    if (cached != nullptr) return cached;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_status_addr[dev].load(std::memory_order_relaxed) == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
        g_status_addr[dev].store(static_cast<unsigned int*>(p), std::memory_order_release);
    }
    return g_status_addr[dev].load(std::memory_order_relaxed);
}

void set_last_error(const char* msg) { t_last_error = msg ? msg : ""; }

}  // namespace attn

using namespace attn;

extern "C" {

const char* attn_status_string(attn_status_t s) {
    switch (s) {
        case ATTN_OK: return "ok";
        case ATTN_ERR_INVALID_ARG: return "invalid argument";
        case ATTN_ERR_UNSUPPORTED: return "unsupported configuration";
        case ATTN_ERR_CUDA: return "CUDA error";
        case ATTN_ERR_TIMEOUT: return "a bounded wait inside a kernel timed out";
    }
    return "unknown status";
}

const char* attn_last_error(void) { return t_last_error.c_str(); }

int attn_version(void) { return 10000; }

attn_status_t attn_status_detail(unsigned int out[4]) {
    t_last_error.clear();
    if (!out) return fail(ATTN_ERR_INVALID_ARG, "null output");
    unsigned int* status = device_status_word();
    if (!status) return fail(ATTN_ERR_CUDA, "cannot resolve the device status word");
    cudaError_t e = cudaMemcpy(out, status, 4 * sizeof(unsigned int), cudaMemcpyDeviceToHost);
    return e == cudaSuccess ? ATTN_OK : cuda_fail(e, "status word read");
}

attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv,
                       int n_q, int n_kv, int d, float scale, int causal, const uint8_t* key_mask,
                       attn_dtype_t dtype, void* stream) {
    t_last_error.clear();
    if (B <= 0 || H <= 0 || H_kv <= 0 || n_q < 0 || n_kv < 0 || d <= 0)
        return fail(ATTN_ERR_INVALID_ARG, "sizes must be positive (B=%d H=%d H_kv=%d d=%d) and n_q, n_kv >= 0", B, H,
                    H_kv, d);
    if (H % H_kv != 0) return fail(ATTN_ERR_INVALID_ARG, "H (%d) must be a multiple of H_kv (%d)", H, H_kv);
    if (causal != 0 && causal != 1) return fail(ATTN_ERR_INVALID_ARG, "causal must be 0 or 1");
    if (dtype != ATTN_DTYPE_F32 && dtype != ATTN_DTYPE_BF16 && dtype != ATTN_DTYPE_BF16_F32OUT)
        return fail(ATTN_ERR_INVALID_ARG, "unknown dtype");
    const bool bf16_in = dtype != ATTN_DTYPE_F32;
    if (!std::isfinite(scale) || !(scale > 0.f))
        return fail(ATTN_ERR_UNSUPPORTED, "scale must be finite and positive");
    if (bf16_in && d != 64 && d != 128)
        return fail(ATTN_ERR_UNSUPPORTED, "bf16 head dim %d not in {64, 128}", d);
    if (bf16_in && key_mask != nullptr && B > 4096)
        return fail(ATTN_ERR_UNSUPPORTED, "bf16 with a key mask supports B <= 4096 (got %d)", B);
    if (dtype == ATTN_DTYPE_F32 && d != 32 && d != 64 && d != 96 && d != 128)
        return fail(ATTN_ERR_UNSUPPORTED, "fp32 head dim %d not in {32, 64, 96, 128}", d);
    const long long rows = (long long)B * H * n_q;
    if ((long long)B * H * n_q * d > (1ll << 40) || (long long)B * H_kv * n_kv * d > (1ll << 40) ||
        n_q > (1 << 30) || n_kv > (1 << 30))
        return fail(ATTN_ERR_UNSUPPORTED, "problem too large");
    if (n_q == 0) return ATTN_OK;
    if (!q || !o || (n_kv > 0 && (!k || !v))) return fail(ATTN_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned(q, 16) || !aligned(o, 16) || (n_kv > 0 && (!aligned(k, 16) || !aligned(v, 16))) ||
        (lse && !aligned(lse, 4)))
        return fail(ATTN_ERR_INVALID_ARG, "q, k, v, o must be 16-byte aligned and lse 4-byte aligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int esize = dtype == ATTN_DTYPE_BF16 ? 2 : 4;  // bytes per element of O
    if (n_kv == 0) {
        fill_empty_rows<<<256, 256, 0, st>>>(o, lse, (size_t)rows, d, esize);
        cudaError_t e = cudaGetLastError();
        return e == cudaSuccess ? ATTN_OK : cuda_fail(e, "fill_empty_rows launch");
    }
    unsigned int* status = device_status_word();
    if (!status) return fail(ATTN_ERR_CUDA, "cannot resolve the device status word");
    FwdArgs a{q, k, v, o, lse, key_mask, B, H, H_kv, n_q, n_kv, d, scale, causal,
              dtype == ATTN_DTYPE_BF16_F32OUT ? 1 : 0};
    cudaError_t e;
    if (dtype == ATTN_DTYPE_F32) {
        e = launch_fwd_f32(a, status, st);
        return e == cudaSuccess ? ATTN_OK : cuda_fail(e, "fp32 forward launch");
    }
    CUtensorMap tq, tk, tv;
    if (!encode_rows_map(&tq, q, d, n_q, H, B, 128) || !encode_rows_map(&tk, k, d, n_kv, H_kv, B, 128) ||
        !encode_rows_map(&tv, v, d, n_kv, H_kv, B, 128))
        return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    e = launch_fwd_bf16_sm100(a, tq, tk, tv, status, st);
    return e == cudaSuccess ? ATTN_OK : cuda_fail(e, "bf16 tcgen05 forward launch");
}

size_t attn_bwd_workspace_bytes(int B, int H, int n_q) {
    if (B <= 0 || H <= 0 || n_q < 0) return 0;
    const size_t rows = (size_t)B * H * (size_t)((n_q + 127) / 128 * 128);
    const size_t bytes = 2 * align_up(rows * sizeof(float), 256);
    return bytes == 0 ? 256 : bytes;
}

attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* d_o,
                       const float* lse, void* dq, void* dk, void* dv, int B, int H, int H_kv, int n_q, int n_kv,
                       int d, float scale, int causal, const uint8_t* key_mask, void* workspace,
                       size_t workspace_bytes, void* stream) {
    t_last_error.clear();
    if (B <= 0 || H <= 0 || H_kv <= 0 || n_q < 0 || n_kv < 0 || d <= 0)
        return fail(ATTN_ERR_INVALID_ARG, "B, H, H_kv, d must be positive and n_q, n_kv >= 0");
    if (H % H_kv != 0) return fail(ATTN_ERR_INVALID_ARG, "H (%d) must be a multiple of H_kv (%d)", H, H_kv);
    if (causal != 0 && causal != 1) return fail(ATTN_ERR_INVALID_ARG, "causal must be 0 or 1");
    if (d != 64 && d != 128) return fail(ATTN_ERR_UNSUPPORTED, "backward head dim %d not in {64, 128}", d);
    if (!std::isfinite(scale) || !(scale > 0.f))
        return fail(ATTN_ERR_UNSUPPORTED, "scale must be finite and positive");
    if ((long long)B * H * n_q * d > (1ll << 40) || (long long)B * H_kv * n_kv * d > (1ll << 40) ||
        n_q > (1 << 30) || n_kv > (1 << 30))
        return fail(ATTN_ERR_UNSUPPORTED, "problem too large");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (n_q == 0 || n_kv == 0) {
        // nothing contributes: the gradients that exist are zero
        if (n_q > 0 && !dq) return fail(ATTN_ERR_INVALID_ARG, "null tensor pointer");
        if (n_kv > 0 && (!dk || !dv)) return fail(ATTN_ERR_INVALID_ARG, "null tensor pointer");
        cudaError_t e = cudaSuccess;
        if (n_q > 0) e = cudaMemsetAsync(dq, 0, (size_t)B * H * n_q * d * 2, st);
        if (e == cudaSuccess && n_kv > 0) e = cudaMemsetAsync(dk, 0, (size_t)B * H_kv * n_kv * d * 2, st);
        if (e == cudaSuccess && n_kv > 0) e = cudaMemsetAsync(dv, 0, (size_t)B * H_kv * n_kv * d * 2, st);
        return e == cudaSuccess ? ATTN_OK : cuda_fail(e, "zero gradients");
    }
    if (!q || !k || !v || !o || !d_o || !lse || !dq || !dk || !dv)
        return fail(ATTN_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(d_o, 16) ||
        !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(lse, 4))
        return fail(ATTN_ERR_INVALID_ARG, "tensors must be 16-byte aligned and lse 4-byte aligned");
    const size_t need = attn_bwd_workspace_bytes(B, H, n_q);
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < need)
        return fail(ATTN_ERR_INVALID_ARG, "workspace must be 256-byte aligned and hold %zu bytes (got %zu)", need,
                    workspace_bytes);
    unsigned int* status = device_status_word();
    if (!status) return fail(ATTN_ERR_CUDA, "cannot resolve the device status word");
    BwdArgs a{};
    a.q = q;
    a.k = k;
    a.v = v;
    a.o = o;
    a.d_o = d_o;
    a.lse = lse;
    a.dq = dq;
    a.dk = dk;
    a.dv = dv;
    a.key_mask = key_mask;
    a.B = B;
    a.H = H;
    a.H_kv = H_kv;
    a.n_q = n_q;
    a.n_kv = n_kv;
    a.d = d;
    a.n_q_pad = (n_q + 127) / 128 * 128;
    a.scale = scale;
    a.causal = causal;
    a.ws_l2 = static_cast<float*>(workspace);
    a.ws_dd = reinterpret_cast<float*>(static_cast<char*>(workspace) + need / 2);
    CUtensorMap tq, tk, tv, tdo;
    if (!encode_rows_map(&tq, q, d, n_q, H, B, 64) || !encode_rows_map(&tdo, d_o, d, n_q, H, B, 64) ||
        !encode_rows_map(&tk, k, d, n_kv, H_kv, B, 64) || !encode_rows_map(&tv, v, d, n_kv, H_kv, B, 64))
        return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    cudaError_t e = launch_bwd(a, tq, tk, tv, tdo, status, st);
    return e == cudaSuccess ? ATTN_OK : cuda_fail(e, "backward launch");
}

attn_status_t attn_fwd_fp8(const void* q, const void* k, const void* v, const float* q_descale,
                           const float* k_descale, const float* v_descale, void* o, float* lse, int B, int H, int H_kv,
                           int n_q, int n_kv, int d, float scale, int causal, const uint8_t* key_mask, int o_f32,
                           void* stream) {
    t_last_error.clear();
    if (B <= 0 || H <= 0 || H_kv <= 0 || n_q < 0 || n_kv < 0 || d <= 0)
        return fail(ATTN_ERR_INVALID_ARG, "B, H, H_kv, d must be positive and n_q, n_kv >= 0");
    if (H % H_kv != 0) return fail(ATTN_ERR_INVALID_ARG, "H (%d) must be a multiple of H_kv (%d)", H, H_kv);
    if (causal != 0 && causal != 1) return fail(ATTN_ERR_INVALID_ARG, "causal must be 0 or 1");
    if (o_f32 != 0 && o_f32 != 1) return fail(ATTN_ERR_INVALID_ARG, "o_f32 must be 0 or 1");
    if (d != 128) return fail(ATTN_ERR_UNSUPPORTED, "FP8 head dim %d: only 128", d);
    if (!std::isfinite(scale) || !(scale > 0.f))
        return fail(ATTN_ERR_UNSUPPORTED, "scale must be finite and positive");
    if (key_mask != nullptr && B > 4096)
        return fail(ATTN_ERR_UNSUPPORTED, "a key mask supports B <= 4096 (got %d)", B);
    if ((long long)B * H * n_q * d > (1ll << 40) || (long long)B * H_kv * n_kv * d > (1ll << 40) ||
        n_q > (1 << 30) || n_kv > (1 << 30))
        return fail(ATTN_ERR_UNSUPPORTED, "problem too large");
    if (n_q == 0) return ATTN_OK;
    if (!q || !o || !q_descale || (n_kv > 0 && (!k || !v || !k_descale || !v_descale)))
        return fail(ATTN_ERR_INVALID_ARG, "null tensor or descale pointer");
    if (!aligned(q, 16) || !aligned(o, 16) || (n_kv > 0 && (!aligned(k, 16) || !aligned(v, 16))) ||
        (lse && !aligned(lse, 4)) || !aligned(q_descale, 4) || (n_kv > 0 && (!aligned(k_descale, 4) ||
                                                                             !aligned(v_descale, 4))))
        return fail(ATTN_ERR_INVALID_ARG, "q, k, v, o must be 16-byte aligned and lse and the descales 4-byte aligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const long long rows = (long long)B * H * n_q;
    if (n_kv == 0) {
        fill_empty_rows<<<256, 256, 0, st>>>(o, lse, (size_t)rows, d, o_f32 ? 4 : 2);
        cudaError_t e = cudaGetLastError();
        return e == cudaSuccess ? ATTN_OK : cuda_fail(e, "fill_empty_rows launch");
    }
    unsigned int* status = device_status_word();
    if (!status) return fail(ATTN_ERR_CUDA, "cannot resolve the device status word");
    FwdArgs a{q, k, v, o, lse, key_mask, B, H, H_kv, n_q, n_kv, d, scale, causal, o_f32};
    a.fp8 = 1;
    a.q_descale = q_descale;
    a.k_descale = k_descale;
    a.v_descale = v_descale;
    CUtensorMap tq, tk, tv;
    if (!encode_rows_map_u8(&tq, q, d, n_q, H, B, 128) || !encode_rows_map_u8(&tk, k, d, n_kv, H_kv, B, 128) ||
        !encode_rows_map_u8(&tv, v, d, n_kv, H_kv, B, 128))
        return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    cudaError_t e = launch_fwd_bf16_sm100(a, tq, tk, tv, status, st);
    return e == cudaSuccess ? ATTN_OK : cuda_fail(e, "fp8 tcgen05 forward launch");
}

attn_status_t attn_prefill_paged(const void* q, const void* k_pages, const void* v_pages,
                                 const int32_t* block_table, const int32_t* seq_lens, int num_seqs, int H, int H_kv,
                                 int n_q, int d, int page_size, int max_pages_per_seq, int num_pages, float scale,
                                 int causal, attn_dtype_t dtype, void* o, float* lse, void* stream) {
    t_last_error.clear();
    if (num_seqs < 0 || H <= 0 || H_kv <= 0 || n_q < 0 || d <= 0 || page_size <= 0 || max_pages_per_seq <= 0 ||
        num_pages <= 0)
        return fail(ATTN_ERR_INVALID_ARG, "sizes must be positive (num_seqs, n_q >= 0)");
    if (H % H_kv != 0) return fail(ATTN_ERR_INVALID_ARG, "H (%d) must be a multiple of H_kv (%d)", H, H_kv);
    if (causal != 0 && causal != 1) return fail(ATTN_ERR_INVALID_ARG, "causal must be 0 or 1");
    if (dtype != ATTN_DTYPE_BF16 && dtype != ATTN_DTYPE_BF16_F32OUT)
        return fail(ATTN_ERR_INVALID_ARG, "dtype must be ATTN_DTYPE_BF16 or ATTN_DTYPE_BF16_F32OUT");
    if (d != 64 && d != 128) return fail(ATTN_ERR_UNSUPPORTED, "head dim %d not in {64, 128}", d);
    if (page_size != 16) return fail(ATTN_ERR_UNSUPPORTED, "page size %d: the paged prefill takes 16-token pages",
                                     page_size);
    if (!std::isfinite(scale) || !(scale > 0.f))
        return fail(ATTN_ERR_UNSUPPORTED, "scale must be finite and positive");
    if ((long long)num_pages * page_size * H_kv * d > (1ll << 40) || (long long)num_seqs * H * n_q * d > (1ll << 40) ||
        (long long)max_pages_per_seq * page_size > (1 << 30))
        return fail(ATTN_ERR_UNSUPPORTED, "problem too large");
    if (num_seqs == 0 || n_q == 0) return ATTN_OK;
    if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !o) return fail(ATTN_ERR_INVALID_ARG, "null pointer");
    if (!aligned(q, 16) || !aligned(k_pages, 16) || !aligned(v_pages, 16) || !aligned(o, 16) ||
        !aligned(block_table, 4) || !aligned(seq_lens, 4) || (lse && !aligned(lse, 4)))
        return fail(ATTN_ERR_INVALID_ARG, "misaligned pointer");
    unsigned int* status = device_status_word();
    if (!status) return fail(ATTN_ERR_CUDA, "cannot resolve the device status word");
    FwdArgs a{q, k_pages, v_pages, o, lse, nullptr, num_seqs, H, H_kv, n_q, max_pages_per_seq * page_size, d, scale,
              causal, dtype == ATTN_DTYPE_BF16_F32OUT ? 1 : 0, block_table, seq_lens, max_pages_per_seq, num_pages};
    CUtensorMap tq, tk, tv;
    if (!encode_rows_map(&tq, q, d, n_q, H, num_seqs, 128) ||
        !encode_pages_map(&tk, k_pages, d, H_kv, page_size, num_pages) ||
        !encode_pages_map(&tv, v_pages, d, H_kv, page_size, num_pages))
        return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    cudaError_t e = launch_fwd_bf16_sm100(a, tq, tk, tv, status, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ATTN_OK : cuda_fail(e, "paged prefill launch");
}

size_t attn_decode_workspace_bytes(int num_seqs, int H, int H_kv, int d, int max_seq_len, int split_tokens) {
    DecodeLayout L;
    if (!decode_layout(num_seqs, H, H_kv, d, max_seq_len, split_tokens, &L)) return 0;
    return L.bytes;
}

attn_status_t attn_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                                const int32_t* block_table, const int32_t* seq_lens, int num_seqs, int H, int H_kv,
                                int d, int page_size, int max_pages_per_seq, int num_pages, int max_seq_len,
                                int split_tokens, float scale, void* workspace, size_t workspace_bytes, void* o,
                                float* lse, void* stream) {
    t_last_error.clear();
    if (num_seqs < 0 || H <= 0 || H_kv <= 0 || d <= 0 || page_size <= 0 || max_pages_per_seq <= 0 ||
        num_pages <= 0 || max_seq_len < 0 || split_tokens < ATTN_DECODE_ONE_LAUNCH)
        return fail(ATTN_ERR_INVALID_ARG,
                    "sizes must be positive (max_seq_len >= 0; split_tokens >= 0 or ATTN_DECODE_ONE_LAUNCH)");
    const bool one_launch = split_tokens == ATTN_DECODE_ONE_LAUNCH;
    if (one_launch && page_size != 16)
        return fail(ATTN_ERR_UNSUPPORTED, "the single-launch decode takes 16-token pages (got %d)", page_size);
    if (H % H_kv != 0) return fail(ATTN_ERR_INVALID_ARG, "H (%d) must be a multiple of H_kv (%d)", H, H_kv);
    const int G = H / H_kv;
    if (G != 1 && G != 2 && G != 4 && G != 8)
        return fail(ATTN_ERR_UNSUPPORTED, "query heads per kv head %d not in {1, 2, 4, 8}", G);
    if (d != 64 && d != 128) return fail(ATTN_ERR_UNSUPPORTED, "head dim %d not in {64, 128}", d);
    if (!std::isfinite(scale) || !(scale > 0.f))
        return fail(ATTN_ERR_UNSUPPORTED, "scale must be finite and positive");
    if ((long long)max_seq_len > (long long)max_pages_per_seq * page_size)
        return fail(ATTN_ERR_INVALID_ARG, "max_seq_len exceeds max_pages_per_seq * page_size");
    if ((long long)num_pages * page_size * H_kv * d > (1ll << 40))
        return fail(ATTN_ERR_UNSUPPORTED, "page pool too large");
    if (num_seqs == 0) return ATTN_OK;
    if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !o || (!workspace && !one_launch))
        return fail(ATTN_ERR_INVALID_ARG, "null pointer");
    if (!aligned(q, 16) || !aligned(k_pages, 16) || !aligned(v_pages, 16) || !aligned(o, 16) ||
        !aligned(workspace, 16) || !aligned(block_table, 4) || !aligned(seq_lens, 4) || (lse && !aligned(lse, 4)))
        return fail(ATTN_ERR_INVALID_ARG, "misaligned pointer");
    DecodeLayout L;
    if (!decode_layout(num_seqs, H, H_kv, d, max_seq_len, split_tokens, &L))
        return fail(ATTN_ERR_INVALID_ARG, "bad workspace arguments");
    if (!one_launch && workspace_bytes < L.bytes)
        return fail(ATTN_ERR_INVALID_ARG, "workspace of %zu bytes, need %zu", workspace_bytes, L.bytes);
    unsigned int* status = device_status_word();
    if (!status) return fail(ATTN_ERR_CUDA, "cannot resolve the device status word");
    DecodeArgs a{};
    a.q = q;
    a.k_pages = k_pages;
    a.v_pages = v_pages;
    a.block_table = block_table;
    a.seq_lens = seq_lens;
    a.num_seqs = num_seqs;
    a.H = H;
    a.H_kv = H_kv;
    a.d = d;
    a.page_size = page_size;
    a.max_pages = max_pages_per_seq;
    a.num_pages = num_pages;
    a.max_seq_len = max_seq_len;
    a.split_tokens = L.split_tokens;
    a.n_splits = L.n_splits;
    a.scale = scale;
    a.part_ml = static_cast<float*>(workspace);
    a.part_u = reinterpret_cast<float*>(static_cast<char*>(workspace) + L.off_u);
    a.o = o;
    a.lse = lse;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (page_size == 16) {
        // tensor-core path: splits cover whole pages (rounding up only lowers the split count,
        // so the workspace sized for split_tokens still suffices); a negative split count
        // selects the single launch with clusters of -n_splits CTAs
        if (!one_launch) {
            a.split_tokens = (L.split_tokens + 15) / 16 * 16;
            a.n_splits = max_seq_len > 0 ? (max_seq_len + a.split_tokens - 1) / a.split_tokens : 1;
        }
        CUtensorMap tk, tv;
        if (!encode_pages_map(&tk, k_pages, d, H_kv, page_size, num_pages) ||
            !encode_pages_map(&tv, v_pages, d, H_kv, page_size, num_pages))
            return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed for the page pool");
        e = launch_decode_mma(a, tk, tv, status, st);
    } else {
        e = launch_decode(a, status, st);
    }
    return e == cudaSuccess ? ATTN_OK : cuda_fail(e, "paged decode launch");
}

attn_status_t attn_testing_set(unsigned long long wait_limit_ns, unsigned int flags) {
    t_last_error.clear();
    if (flags & ~ATTN_TEST_DROP_FIRST_V) return fail(ATTN_ERR_INVALID_ARG, "unknown test flags 0x%x", flags);
    unsigned int* status = device_status_word();
    if (!status) return fail(ATTN_ERR_CUDA, "cannot resolve the device status word");
    const unsigned int words[4] = {(unsigned int)(wait_limit_ns & 0xffffffffull), (unsigned int)(wait_limit_ns >> 32),
                                   flags, 0u};
    cudaError_t e = cudaMemcpy(status + 4, words, sizeof words, cudaMemcpyHostToDevice);
    return e == cudaSuccess ? ATTN_OK : cuda_fail(e, "test hook write");
}

attn_status_t attn_check_status(void* stream) {
    t_last_error.clear();
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    unsigned int* status = device_status_word();
    if (!status) return fail(ATTN_ERR_CUDA, "cannot resolve the device status word");
    unsigned int words[4] = {0, 0, 0, 0};
    e = cudaMemcpy(words, status, sizeof words, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "status word read");
    const unsigned int word = words[0];
    if (word != 0 || words[1] != 0) {
        const unsigned int zero[4] = {0, 0, 0, 0};
        e = cudaMemcpy(status, zero, sizeof zero, cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return cuda_fail(e, "status word clear");
    }
    if (word & ATTN_DEV_TIMEOUT)
        return fail(ATTN_ERR_TIMEOUT, "device status word 0x%x; first give-up: warp %u site %u block %u parity %u",
                    word, (words[1] >> 8) & 0xFFu, words[1] & 0xFFu, words[2], words[3]);
    if (word & ATTN_DEV_SMEM_LAYOUT)
        return fail(ATTN_ERR_CUDA, "device status word 0x%x (dynamic shared memory too small for the aligned layout)",
                    word);
    if (word & (ATTN_DEV_BAD_PAGE | ATTN_DEV_BAD_LEN | ATTN_DEV_BAD_SCALE))
        return fail(ATTN_ERR_INVALID_ARG, "device status word 0x%x (bad page id, sequence length or FP8 descale)",
                    word);
    return ATTN_OK;
}

}  // extern "C"
