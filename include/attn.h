/*
 * attn.h - C ABI of libattn.so: exact scaled-dot-product attention on B200 (sm_100a).
 *
 * The operation (scaled dot-product attention, "Sviluppo AI ed Algebra Lineare",
 * the SDPA formula softmax(QK^T / sqrt(d_k)) V; one row of it is the object of
 * "Attenzione: softmax online, riscalamento e memoria", section 1):
 *
 *   for batch b, query head h, query row i, with kv head g = h / (H / H_kv):
 *     K_i    = { key j : key_mask[b][j] != 0 (or no mask), and j <= i + n_kv - n_q if causal }
 *     s_j    = scale * <q[b][h][i], k[b][g][j]>
 *     o      = sum_{j in K_i} exp(s_j) v[b][g][j] / sum_{j in K_i} exp(s_j)
 *     lse    = ln sum_{j in K_i} exp(s_j)
 *
 * computed with the blocked online softmax (running maximum, normaliser and
 * unnormalised accumulator rescaled together; same page, section 2), so the
 * score matrix never reaches device memory.  A row whose K_i is empty (fully
 * masked, or causal with n_q > n_kv) gets o = 0 and lse = -inf: the pages
 * leave that 0/0 case to an explicit convention and this is the one taken.
 *
 * Conventions shared by every entry point:
 *   - Every pointer argument is caller-owned DEVICE memory (cudaMalloc or a
 *     framework allocator) on the current CUDA device, unless stated
 *     otherwise.  The library keeps no reference after a call returns.
 *   - All tensors are dense and row-major in the stated shapes (last index
 *     fastest).  bf16 means IEEE bfloat16; fp32 means IEEE binary32.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Calls are asynchronous: they validate, enqueue kernels and
 *     return without synchronising the host.
 *   - Arguments are validated before anything is launched; an invalid or
 *     unsupported call returns an error status and launches nothing.  A
 *     launch failure returns ATTN_ERR_CUDA.  There is no fallback path.
 *   - Problems that only the device can see (a block-table entry outside the
 *     page pool, a sequence length beyond the stated bounds, a bounded wait
 *     inside a kernel that gave up) are recorded in a per-device status word;
 *     attn_check_status() reads and clears it.  Kernels never trap.
 *   - Thread safety: entry points may be called concurrently from several
 *     host threads; they share only the per-device status word.
 *   - The device addresses of the library's own device variables (the status
 *     word, the fixed scratch of attn_decode_paged_static) are looked up once
 *     per device and kept for the life of the process, and so are the kernels'
 *     launch attributes (their shared-memory sizes): do not call the library
 *     on a device after cudaDeviceReset.
 */
#ifndef ATTN_H_
#define ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, inconsistent shapes, bad device data */
    ATTN_ERR_UNSUPPORTED = 2, /* valid request outside what the kernels implement (e.g. head dim) */
    ATTN_ERR_CUDA = 3,        /* a CUDA call or kernel launch failed; see attn_last_error() */
    ATTN_ERR_TIMEOUT = 4      /* a bounded wait inside a kernel gave up (reported by attn_check_status) */
} attn_status_t;

typedef enum {
    ATTN_DTYPE_F32 = 0,         /* q, k, v, o fp32 */
    ATTN_DTYPE_BF16 = 1,        /* q, k, v, o bf16 */
    ATTN_DTYPE_BF16_F32OUT = 2  /* q, k, v bf16; o fp32 (the same arithmetic, without the final bf16 rounding) */
} attn_dtype_t;

/*
 * attn_fwd - prefill / forward attention for a batch of sequences.
 *
 * q    [B, H,    n_q,  d]   input dtype       (16-byte aligned)
 * k    [B, H_kv, n_kv, d]   input dtype       (16-byte aligned)
 * v    [B, H_kv, n_kv, d]   input dtype       (16-byte aligned)
 * o    [B, H,    n_q,  d]   output dtype, written (16-byte aligned)
 * lse  [B, H,    n_q]       fp32, written; may be NULL.  Natural log of the
 *                            sum of exp(scaled score) over the kept keys.
 * key_mask [B, n_kv] uint8, 1 = keep, 0 = exclude, shared by all heads and
 *                            rows of batch b; NULL = keep every key.
 * scale    multiplies q.k (typically 1/sqrt(d)); must be finite and > 0.
 * causal   0 or 1; when 1, row i keeps keys j <= i + n_kv - n_q (queries are
 *          the last n_q positions of the sequence).
 * H % H_kv must be 0; query head h reads kv head h / (H / H_kv).
 *
 * Supported: dtype BF16 / BF16_F32OUT with d in {64, 128} (tensor cores, fp32
 * accumulation; P rounded to bf16 for the second product, l summed from those
 * rounded weights; with a key_mask, B <= 4096); dtype F32 with d in
 * {32, 64, 96, 128} (fp32 FMA throughout).
 * n_q == 0 is a no-op; n_kv == 0 writes o = 0 and lse = -inf.
 */
attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv,
                       int n_q, int n_kv, int d, float scale, int causal, const uint8_t* key_mask,
                       attn_dtype_t dtype, void* stream);

/*
 * attn_fwd_fp8 - attn_fwd on block-scaled FP8 E4M3 inputs ("Sviluppo AI ed Algebra
 * Lineare", the FP8 section on FlashAttention-3, "Quantizzazione a Blocchi e Scaling
 * Algebrico": each block X of rows is stored as X_fp8 with its own scale s_X, the
 * products run on the 8-bit values with fp32 accumulation, and the scales are applied
 * to the accumulators: S_ij = s_Q,i s_K,j (Q_i,fp8 K_j,fp8^T) scale; P is quantised to
 * E4M3 for the second product; O is normalised in fp32 at the end).
 *
 * q, k, v hold E4M3 bit patterns (one byte per element, layouts as attn_fwd).  The
 * blocks are 128 rows of one head (ATTN_FP8_BLOCK): element (b, h, i, c) of q stands
 * for q_descale[b][h][i / 128] * decode(q[b][h][i][c]), and likewise for k and v.
 *   q_descale  [B, H,    ceil(n_q  / 128)] fp32, device memory, each finite and > 0
 *   k_descale  [B, H_kv, ceil(n_kv / 128)] fp32, device memory, each finite and > 0
 *   v_descale  [B, H_kv, ceil(n_kv / 128)] fp32, device memory, each finite and > 0
 * A descale that is not finite and positive gives undefined output and sets the
 * device status word (attn_check_status returns ATTN_ERR_INVALID_ARG).
 * o is bf16 (o_f32 = 0) or fp32 (o_f32 = 1); lse as attn_fwd (may be NULL).
 * key_mask and causal as attn_fwd (with a key mask, B <= 4096).
 * Supported: d = 128; H % H_kv == 0.
 * Rounding: P is rounded to E4M3 (round to nearest) measured 2^8 above the running row
 * maximum and multiplied by v_descale[j] / (the kv head's largest v_descale), <= 1;
 * l for O is summed from those rounded weights (each divided back by that factor) and
 * l for the LSE from the unrounded ones.
 */
#define ATTN_FP8_BLOCK 128
attn_status_t attn_fwd_fp8(const void* q, const void* k, const void* v, const float* q_descale,
                           const float* k_descale, const float* v_descale, void* o, float* lse, int B, int H, int H_kv,
                           int n_q, int n_kv, int d, float scale, int causal, const uint8_t* key_mask, int o_f32,
                           void* stream);

/*
 * attn_decode_workspace_bytes - size of the scratch buffer attn_decode_paged
 * needs for these arguments (split_tokens = 0 selects the library's choice,
 * exactly as attn_decode_paged will; ATTN_DECODE_ONE_LAUNCH needs none and
 * gives 16).  Returns 0 for invalid arguments.  The
 * size is computed for split_tokens as given; with 16-token pages the call
 * rounds a split up to whole pages, which only lowers the number of partial
 * states, so this size is then an upper bound (pass a multiple of 16 for the
 * exact figure).
 */
size_t attn_decode_workspace_bytes(int num_seqs, int H, int H_kv, int d, int max_seq_len, int split_tokens);

/*
 * attn_decode_paged - one query token per sequence against a paged KV cache.
 *
 * The cache is a pool of fixed-size pages and a block table mapping each
 * sequence's logical page to a physical page ("Kernel di attenzione rapida e
 * fusione degli operatori", section "Attenzione di tipo FlashAttention e
 * attenzione paginata").  Token t of sequence s is slot t % page_size of page
 * block_table[s][t / page_size].  The work is split over groups of
 * split_tokens tokens; each group writes a partial (m, l, u) state to the
 * workspace and a second kernel merges them with the disjoint-set rule of
 * "Attenzione: softmax online, riscalamento e memoria", section 4.
 *
 * q           [num_seqs, H, d] bf16                       (16-byte aligned)
 * k_pages     [num_pages, page_size, H_kv, d] bf16        (16-byte aligned)
 * v_pages     [num_pages, page_size, H_kv, d] bf16        (16-byte aligned)
 * block_table [num_seqs, max_pages_per_seq] int32 physical page ids
 * seq_lens    [num_seqs] int32, each in [0, max_seq_len]
 * max_seq_len host-side bound on every seq_lens entry (sizes the grid);
 *             must be <= max_pages_per_seq * page_size
 * split_tokens tokens per split (>= 1), or 0 for the library's choice; with
 *             16-token pages it is rounded up to a multiple of 16 (whole pages).
 *             ATTN_DECODE_ONE_LAUNCH (16-token pages only): one kernel, no
 *             workspace.  The CTAs of each (sequence, kv head) form a
 *             thread-block cluster (two CTAs, one for a single page), split the
 *             sequence's pages into equal contiguous shares, and merge their
 *             partial states on chip through distributed shared memory (same
 *             rule, fixed order), so no partial state is written to memory and
 *             no merge kernel runs.  The split path is faster on large batches.
 * workspace   device scratch of at least attn_decode_workspace_bytes(...)
 *             bytes, 16-byte aligned; its contents on entry do not matter
 *             (may be NULL with ATTN_DECODE_ONE_LAUNCH)
 * o           [num_seqs, H, d] bf16, written              (16-byte aligned)
 * lse         [num_seqs, H] fp32, written; may be NULL
 * Supported: d in {64, 128}; H / H_kv in {1, 2, 4, 8}; any page_size >= 1
 * (16-token pages run on the tensor cores with TMA page copies, other sizes on
 * the CUDA cores).
 * A sequence of length 0 gets o = 0 and lse = -inf.  Page ids outside
 * [0, num_pages) are skipped and a length beyond max_seq_len is clamped; both
 * set the device status word (attn_check_status returns ATTN_ERR_INVALID_ARG).
 */
#define ATTN_DECODE_ONE_LAUNCH (-1)
attn_status_t attn_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                                const int32_t* block_table, const int32_t* seq_lens, int num_seqs, int H, int H_kv,
                                int d, int page_size, int max_pages_per_seq, int num_pages, int max_seq_len,
                                int split_tokens, float scale, void* workspace, size_t workspace_bytes, void* o,
                                float* lse, void* stream);

/*
 * attn_prefill_paged - a block of n_q query tokens per sequence against the
 * sequence's keys and values in a paged KV cache (chunked prefill over the cache
 * of "Kernel di attenzione rapida e fusione degli operatori", section
 * "Attenzione di tipo FlashAttention e attenzione paginata"), computed with the
 * blocked online softmax of attn_fwd.
 *
 * Sequence s holds seq_lens[s] tokens; token t lives in slot t % 16 of page
 * block_table[s][t / 16].  The query rows are the sequence's last n_q positions,
 * so with causal = 1 query i keeps the keys t <= i + seq_lens[s] - n_q (rows with
 * no key, when seq_lens[s] < n_q, get o = 0 and lse = -inf); with causal = 0 it
 * keeps all seq_lens[s] keys.
 *
 * q           [num_seqs, H, n_q, d] bf16                  (16-byte aligned)
 * k_pages     [num_pages, 16, H_kv, d] bf16               (16-byte aligned)
 * v_pages     [num_pages, 16, H_kv, d] bf16               (16-byte aligned)
 * block_table [num_seqs, max_pages_per_seq] int32 physical page ids
 * seq_lens    [num_seqs] int32, each in [0, max_pages_per_seq * 16]
 * dtype       ATTN_DTYPE_BF16 (o bf16) or ATTN_DTYPE_BF16_F32OUT (o fp32: the
 *             same arithmetic without the final bf16 rounding)
 * o           [num_seqs, H, n_q, d] bf16 or fp32 per dtype, written (16-byte aligned)
 * lse         [num_seqs, H, n_q] fp32, written; may be NULL
 * scale       multiplies q.k; finite and > 0.
 * Supported: page_size 16; d in {64, 128}; H % H_kv == 0.  Slots past a
 * sequence's end may hold anything (NaN included): they never reach o.  A page
 * id outside [0, num_pages) for a token of the sequence is replaced by page 0 and
 * sets the device status word (attn_check_status returns ATTN_ERR_INVALID_ARG);
 * that sequence's output is then meaningless.  A length outside
 * [0, max_pages_per_seq * 16] is clamped.
 */
attn_status_t attn_prefill_paged(const void* q, const void* k_pages, const void* v_pages,
                                 const int32_t* block_table, const int32_t* seq_lens, int num_seqs, int H, int H_kv,
                                 int n_q, int d, int page_size, int max_pages_per_seq, int num_pages, float scale,
                                 int causal, attn_dtype_t dtype, void* o, float* lse, void* stream);

/*
 * attn_bwd - gradients of attn_fwd (bf16) with recomputation: dq, dk, dv from
 * q, k, v, the forward's o and lse, and the output gradient d_o, without the
 * n_q x n_kv weight matrix in memory ("Sviluppo AI ed Algebra Lineare", section "Ricalcolo
 * nel Backward Pass (Recomputation)": only the forward's row statistics are
 * kept and the score and weight blocks are recomputed tile by tile).  With
 * P = softmax over the kept keys of scale * q.k (the keys attn_fwd keeps for the
 * same causal and key_mask), they are the gradients of sum(d_o * o):
 *   dv_j = sum_i P_ij d_o_i,   dS_ij = P_ij (d_o_i.v_j - d_o_i.o_i),
 *   dq_i = scale sum_j dS_ij k_j,   dk_j = scale sum_i dS_ij q_i,
 * with dk and dv summed over the H / H_kv query heads of each kv head.
 *
 * q, o, d_o   [B, H, n_q, d] bf16                    (16-byte aligned)
 * k, v        [B, H_kv, n_kv, d] bf16                (16-byte aligned)
 * lse         [B, H, n_q] fp32, natural log, as attn_fwd writes it (-inf for a
 *             row with no kept key; such rows add nothing)
 * dq          [B, H, n_q, d] bf16, written           (16-byte aligned)
 * dk, dv      [B, H_kv, n_kv, d] bf16, written       (16-byte aligned)
 * key_mask    [B, n_kv] uint8, nonzero = keep, or NULL
 * workspace   device memory of at least attn_bwd_workspace_bytes(B, H, n_q)
 *             bytes, 256-byte aligned, owned by the caller; overwritten.
 * scale, causal as for attn_fwd.  Supported: d in {64, 128}, H % H_kv == 0.
 * Errors are returned before any launch.  Every output element is written
 * (zeros where no key or no query contributes).  The result is deterministic
 * (fixed summation order, no atomics).  The call allocates nothing and does
 * not synchronise the host.
 */
size_t attn_bwd_workspace_bytes(int B, int H, int n_q);
attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* d_o,
                       const float* lse, void* dq, void* dk, void* dv, int B, int H, int H_kv, int n_q, int n_kv,
                       int d, float scale, int causal, const uint8_t* key_mask, void* workspace,
                       size_t workspace_bytes, void* stream);

/*
 * attn_decode_paged_static - attn_decode_paged for callers that cannot allocate
 * device memory.  (No counterpart in the pages: this is a deployment aid.)
 *
 * Some callers cannot call cudaMalloc or hand over a workspace: code running
 * inside a host callback or an allocator's own path, under a device-memory
 * budget that must not change, or in a plugin whose host framework owns every
 * allocation.  This entry point takes the same arguments as attn_decode_paged
 * minus the workspace, and keeps the split-KV partial states in one fixed
 * scratch array of 32 MiB (33554432 bytes) compiled into the library; every
 * GPU that loads the library holds that array until the process exits.  It
 * allocates nothing (no cudaMalloc, no cudaFree, no allocating library call)
 * and launches the same kernels as attn_decode_paged.
 *
 * Limit: the arguments must need at most 32 MiB of partial states, i.e.
 * attn_decode_workspace_bytes(num_seqs, H, H_kv, d, max_seq_len, split_tokens)
 * <= 33554432 (64 sequences x 32 heads up to 8192 tokens at d = 128 fit with
 * the default split); larger requests return ATTN_ERR_INVALID_ARG with the
 * sizes in attn_last_error() and launch nothing.
 * Set-up: the first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current), which may load the
 * library's code onto the device; make that first call before any stream
 * capture.  The address is kept for the life of the process, so a device
 * that has been through cudaDeviceReset must not be given to this call again.
 * Sharing: every call on a device uses the same array, which keeps the last
 * call's contents.  Nothing in it needs to start at zero (each call writes
 * every partial state it later reads).  Calls whose kernels overlap on the GPU
 * (different streams, or host threads without ordering) race on the array
 * and give wrong results: order them on one stream.
 */
attn_status_t attn_decode_paged_static(const void* q, const void* k_pages, const void* v_pages,
                                       const int32_t* block_table, const int32_t* seq_lens, int num_seqs, int H,
                                       int H_kv, int d, int page_size, int max_pages_per_seq, int num_pages,
                                       int max_seq_len, int split_tokens, float scale, void* o, float* lse,
                                       void* stream);

/* attn_status_string - static English description of a status code. */
const char* attn_status_string(attn_status_t status);

/* attn_last_error - detail of the last failed call on this host thread
 * (validation message or CUDA error string); "" if none.  Thread-local storage. */
const char* attn_last_error(void);

/*
 * attn_check_status - synchronise `stream`, then read and clear the current
 * device's status word.  Returns ATTN_ERR_TIMEOUT if a kernel's bounded wait
 * gave up, ATTN_ERR_INVALID_ARG if a kernel met bad device data (page id or
 * sequence length), ATTN_ERR_CUDA if the stream reports an error, else ATTN_OK.
 */
attn_status_t attn_check_status(void* stream);

/* attn_version - library version as major*10000 + minor*100 + patch. */
int attn_version(void);

/*
 * attn_status_detail - copy the current device's four status words without
 * clearing them: [0] the flag bits attn_check_status maps to a status;
 * [1] 0x80000000 | warp << 8 | wait-site code of the first bounded wait that
 * gave up (0 if none); [2] that CTA's linear block index; [3] the phase parity
 * it waited for.  `out` is host memory.  Does not synchronise any stream.
 */
attn_status_t attn_status_detail(unsigned int out[4]);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_H_ */
