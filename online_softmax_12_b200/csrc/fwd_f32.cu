// fp32 forward attention on the CUDA cores (SIMT FMA).
//
// The same blocked online softmax as the tensor-core kernel (running maximum m,
// normaliser l and unnormalised accumulator u per query row, all three rescaled
// together by exp(m_old - m_new) before a key block is added: "Attenzione:
// softmax online, riscalamento e memoria", section 2; the two-block merge of
// "Sviluppo AI ed Algebra Lineare", section "Online Softmax"), in fp32 FMA so
// that the fp32 tolerance holds (TF32 tensor cores would round the scores to
// 10 mantissa bits).
//
// One CTA = 128 threads = 16 query rows of one (batch, head).  Key/value blocks
// of 64 rows are staged in shared memory through a two-stage cp.async pipeline
// (block t + 1 loads while block t is computed), so the kernel waits for global
// memory once, not once per block.  Each row is served by 8 consecutive lanes:
// for the scores every lane takes 8 of the 64 keys; for the output every lane
// owns D/8 columns.  Row maxima and sums are reduced with 8-lane shuffles.
// Scores are kept in base-2 units (scale * log2(e) folded in), so every
// exponential is one ex2 instruction; the log-sum-exp is converted back to the
// natural log of the scaled scores at the end.
#include <cfloat>
#include <climits>
#include <cmath>

#include "internal.h"

namespace attn {
namespace {

constexpr int kRows = 16;     // query rows per CTA
constexpr int kKeys = 64;     // keys per shared-memory block
constexpr int kThreads = 128;

constexpr int kStages = 2;    // key/value blocks in flight
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct F32Smem {
    static constexpr int kPad = D + 4;  // 16-byte aligned rows, conflict-free float4 reads
    float q[kRows][kPad];
    float k[kStages][kKeys][kPad];
    float v[kStages][kKeys][D];
    float p[kRows][kKeys];
    unsigned char keep[kStages][kKeys];
};

// 16-byte asynchronous copy global -> shared; with valid = false nothing is read
// and the 16 bytes are zero-filled.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ float ex2f(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <int D>
__global__ void __launch_bounds__(kThreads) fwd_f32_kernel(FwdArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    F32Smem<D>& s = *reinterpret_cast<F32Smem<D>*>(smem_raw);

    const int tid = threadIdx.x;
    const int row0 = blockIdx.x * kRows;
    const int h = blockIdx.y, b = blockIdx.z;
    const int g = h / (a.H / a.H_kv);
    const float* __restrict__ q = static_cast<const float*>(a.q) + ((size_t)(b * a.H + h) * a.n_q) * D;
    const float* __restrict__ kbase = static_cast<const float*>(a.k) + ((size_t)(b * a.H_kv + g) * a.n_kv) * D;
    const float* __restrict__ vbase = static_cast<const float*>(a.v) + ((size_t)(b * a.H_kv + g) * a.n_kv) * D;
    const int offset = a.n_kv - a.n_q;  // bottom-right causal alignment

    // stage the 16 query rows (zeros past n_q)
    for (int e = tid * 4; e < kRows * D; e += kThreads * 4) {
        const int r = e / D, c = e % D;
        float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
        if (row0 + r < a.n_q) val = *reinterpret_cast<const float4*>(q + (size_t)(row0 + r) * D + c);
        *reinterpret_cast<float4*>(&s.q[r][c]) = val;
    }

    const int r = tid / 8;       // this lane's query row within the CTA
    const int lane8 = tid % 8;   // position among the row's 8 lanes
    const int row = row0 + r;
    constexpr int kChunks = D / 32;  // float4 chunks of the output row per lane

    float m_run = -INFINITY, l_run = 0.f;
    float acc[kChunks][4];
#pragma unroll
    for (int i = 0; i < kChunks; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

    int kv_end = a.n_kv;
    if (a.causal) kv_end = min(kv_end, row0 + kRows + offset);  // last row of the CTA sees j <= row + offset
    const int row_limit = a.causal ? row + offset : INT_MAX;    // this row sees keys j <= row_limit
    const int n_blocks = kv_end > 0 ? (kv_end + kKeys - 1) / kKeys : 0;
    const float sl2 = a.scale * kLog2e;

    // stage block t (keys t*64 ...) into stage t % 2: K, V rows by cp.async, keep flags by plain stores
    auto load_block = [&](int t) {
        const int st = t % kStages, n0 = t * kKeys;
        for (int e = tid * 4; e < kKeys * D; e += kThreads * 4) {
            const int j = e / D, c = e % D;
            const bool ok = n0 + j < a.n_kv;
            const size_t off = ok ? (size_t)(n0 + j) * D + c : 0;
            cp_async16(&s.k[st][j][c], kbase + off, ok);
            cp_async16(&s.v[st][j][c], vbase + off, ok);
        }
        if (tid < kKeys) {
            const int j = n0 + tid;
            s.keep[st][tid] = (j < a.n_kv) && (a.key_mask == nullptr || a.key_mask[(size_t)b * a.n_kv + j] != 0);
        }
        cp_async_commit();
    };
    if (n_blocks > 0) load_block(0);

    for (int t = 0; t < n_blocks; ++t) {
        const int st = t % kStages, n0 = t * kKeys;
        if (t + 1 < n_blocks) {
            load_block(t + 1);   // its stage was released by the barrier at the end of block t - 1
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();         // block t's rows (and the query rows) visible to every thread

        // scores of this lane's 8 keys: j = lane8 + 8 t, in base-2 units
        float sc[8];
        float blk_max = -INFINITY;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int jj = lane8 + 8 * u;
            float dot = 0.f;
#pragma unroll
            for (int c = 0; c < D; c += 4) {
                const float4 qa = *reinterpret_cast<const float4*>(&s.q[r][c]);
                const float4 ka = *reinterpret_cast<const float4*>(&s.k[st][jj][c]);
                dot = fmaf(qa.x, ka.x, dot);
                dot = fmaf(qa.y, ka.y, dot);
                dot = fmaf(qa.z, ka.z, dot);
                dot = fmaf(qa.w, ka.w, dot);
            }
            const bool keep = s.keep[st][jj] && (n0 + jj <= row_limit);
            sc[u] = keep ? dot * sl2 : -INFINITY;
            blk_max = fmaxf(blk_max, sc[u]);
        }
#pragma unroll
        for (int off = 4; off >= 1; off >>= 1) blk_max = fmaxf(blk_max, __shfl_xor_sync(0xffffffffu, blk_max, off));

        const float m_new = fmaxf(m_run, blk_max);
        // no key kept so far: keep every weight at exactly zero
        const float base = (m_new == -INFINITY) ? 0.f : m_new;
        const float alpha = ex2f(m_run - base);  // 2^-inf = 0 on the first kept block
        float blk_sum = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const float p = ex2f(sc[u] - base);
            s.p[r][lane8 + 8 * u] = p;
            blk_sum += p;
        }
#pragma unroll
        for (int off = 4; off >= 1; off >>= 1) blk_sum += __shfl_xor_sync(0xffffffffu, blk_sum, off);
        l_run = l_run * alpha + blk_sum;
        m_run = m_new;
        __syncwarp();

        // u <- u * alpha + sum_j p_j v_j over this block
#pragma unroll
        for (int i = 0; i < kChunks; ++i) {
            acc[i][0] *= alpha; acc[i][1] *= alpha; acc[i][2] *= alpha; acc[i][3] *= alpha;
        }
#pragma unroll 4
        for (int j = 0; j < kKeys; ++j) {
            const float p = s.p[r][j];
#pragma unroll
            for (int i = 0; i < kChunks; ++i) {
                const float4 vv = *reinterpret_cast<const float4*>(&s.v[st][j][4 * (lane8 + 8 * i)]);
                acc[i][0] = fmaf(p, vv.x, acc[i][0]);
                acc[i][1] = fmaf(p, vv.y, acc[i][1]);
                acc[i][2] = fmaf(p, vv.z, acc[i][2]);
                acc[i][3] = fmaf(p, vv.w, acc[i][3]);
            }
        }
        __syncthreads();         // stage st fully consumed before block t + 2 loads into it
    }

    if (row < a.n_q) {
        float* o = static_cast<float*>(a.o) + ((size_t)(b * a.H + h) * a.n_q + row) * D;
        const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
#pragma unroll
        for (int i = 0; i < kChunks; ++i) {
            float4 out = make_float4(acc[i][0] * inv, acc[i][1] * inv, acc[i][2] * inv, acc[i][3] * inv);
            *reinterpret_cast<float4*>(o + 4 * (lane8 + 8 * i)) = out;
        }
        if (a.lse != nullptr && lane8 == 0)
            a.lse[(size_t)(b * a.H + h) * a.n_q + row] =
                (l_run > 0.f) ? (m_run + log2f(l_run)) * 0.6931471805599453f : -INFINITY;
    }
}

template <int D>
cudaError_t launch_d(const FwdArgs& a, cudaStream_t stream) {
    const size_t smem = sizeof(F32Smem<D>);
    static std::atomic<unsigned long long> ready{0};
    int dev = 0;
    cudaError_t e = setup_once_per_device(ready, &dev, [smem](int) {
        return cudaFuncSetAttribute(fwd_f32_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    });
    if (e != cudaSuccess) return e;
    dim3 grid((a.n_q + kRows - 1) / kRows, a.H, a.B);
    fwd_f32_kernel<D><<<grid, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_f32(const FwdArgs& a, unsigned int* /*status*/, cudaStream_t stream) {
    switch (a.d) {
        case 32: return launch_d<32>(a, stream);
        case 64: return launch_d<64>(a, stream);
        case 96: return launch_d<96>(a, stream);
        case 128: return launch_d<128>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace attn
