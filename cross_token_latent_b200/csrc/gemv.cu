// Weight-streaming projection for a few rows (M <= 4), the decode shape of single-sequence
// and very small batches: C[M, N] = A[M, K] x W[N, K]^T on CUDA cores.  At these sizes a
// projection is a pass over its weights (2 bytes per multiply-add pair and row of C), so the
// kernel is built to stream W at HBM speed rather than to use the tensor cores:
//   - CTA c owns a contiguous block of weight rows [n0, n1) (a multiple of 32 rows, so that the
//     gate/up and gate/feedback pairs and the 16-column deferred-norm groups stay inside it);
//   - its rows are one contiguous byte range of W, moved into a ring of shared-memory chunks of
//     GV_WARPS rows by 1-D bulk asynchronous copies completing on mbarriers;
//   - the first chunks are requested before the programmatic-launch dependency wait: the
//     weights do not depend on the previous kernel, so their HBM traffic overlaps its tail;
//   - warp w computes row w of every chunk: lanes walk K in 16-byte pieces of the row (shared
//     memory) and of each activation row (read-only global loads), float32 accumulation, one
//     warp reduction per row of C;
//   - the dot products of the CTA's rows are kept in shared memory and the fused epilogue
//     (StoreF32, ResidAdd, SwiGLU, Merge, the deferred norm on both sides) runs over them with
//     the same arithmetic as the tensor-core kernels' epilogues.
// Every mbarrier wait is bounded; on expiry the CTA latches ERR_TIMEOUT, waits (bounded) for
// the copies it issued and returns without storing.
#include "kernels.cuh"
#include "sm100.cuh"

namespace rlt {

namespace {

constexpr int GV_WARPS = 4;                 // warps per CTA = weight rows per chunk
constexpr int GV_MAX_STAGES = 8;
constexpr int GV_RING_BYTES = 96 * 1024;    // two CTAs fit on an SM beside each other
constexpr int GV_MAX_ROWS = 128;            // weight rows per CTA (dots kept in shared memory)

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

template <int MB>
__global__ void __launch_bounds__(GV_WARPS * 32) k_gemv(const bf16* __restrict__ W, const bf16* __restrict__ A,
                                                        int lda, int M, int N, int K, int rows_per_cta, int stages,
                                                        Epi epi, EpiArgs ea, DevHeader* hdr) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    __shared__ uint64_t full[GV_MAX_STAGES];
    __shared__ float res[MB][GV_MAX_ROWS];
    __shared__ float rinv[MB];
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * rows_per_cta;
    const int n1 = min(N, n0 + rows_per_cta);
    const int nrows = n1 - n0;
    const int nchunks = (nrows + GV_WARPS - 1) / GV_WARPS;
    const size_t row_bytes = (size_t)K * 2;
    const size_t chunk_bytes = GV_WARPS * row_bytes;
    const uint64_t lim = ea.wait_ns;
    pdl_trigger();

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) mbar_init(&full[s], 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    int armed = 0;                          // thread 0: chunks whose copies have been issued
    auto issue = [&](int c) {
        const int r0 = c * GV_WARPS;
        const uint32_t bytes = (uint32_t)(min(GV_WARPS, nrows - r0) * row_bytes);
        uint64_t* bar = &full[c % stages];
        mbar_expect_tx(bar, bytes);
        bulk_load(ring + (size_t)(c % stages) * chunk_bytes, W + (size_t)(n0 + r0) * K, bytes, bar);
        armed = c + 1;
    };
    if (threadIdx.x == 0 && !ea.no_loads)
        for (int c = 0; c < min(stages, nchunks); ++c) issue(c);
    pdl_wait();
    if (ea.ss_in && threadIdx.x < M) rinv[threadIdx.x] = deferred_rinv(ea, threadIdx.x);

    const int nv = K / 8;                   // 16-byte pieces per row
    bool ok = true;
    for (int c = 0; c < nchunks && ok; ++c) {
        ok = mbar_wait(&full[c % stages], (uint32_t)((c / stages) & 1), &abort_flag, lim);
        if (!ok) abort_flag = 1;
        const int r = c * GV_WARPS + warp;
        if (ok && r < nrows) {
            const uint4* wrow = reinterpret_cast<const uint4*>(ring + (size_t)(c % stages) * chunk_bytes +
                                                               (size_t)warp * row_bytes);
            float acc[MB];
#pragma unroll
            for (int m = 0; m < MB; ++m) acc[m] = 0.f;
            for (int v = lane; v < nv; v += 32) {
                float w8[8];
                Vec16<bf16>::unpack(wrow[v], w8);
#pragma unroll
                for (int m = 0; m < MB; ++m) {
                    if (m < M) {
                        float a8[8];
                        Vec16<bf16>::unpack(__ldg(reinterpret_cast<const uint4*>(A + (size_t)m * lda) + v), a8);
#pragma unroll
                        for (int i = 0; i < 8; ++i) acc[m] = fmaf(w8[i], a8[i], acc[m]);
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < MB; ++m) {
                const float sum = warp_sum(acc[m]);
                if (lane == 0) res[m][r] = sum;
            }
        }
        ok = __syncthreads_and(ok) && abort_flag == 0;     // every warp is done with the slot
        if (ok && threadIdx.x == 0 && c + stages < nchunks && !ea.no_loads) issue(c + stages);
    }
    if (!ok) {
        if (threadIdx.x == 0) {
            raise_flag(hdr, ERR_TIMEOUT);
            for (int c = armed > stages ? armed - stages : 0; c < armed; ++c)
                mbar_wait(&full[c % stages], (uint32_t)((c / stages) & 1), nullptr, lim);
        }
        return;
    }

    // epilogue over the CTA's rows of C (GEMM columns n0 .. n1-1)
    const int total = M * nrows;
    for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {
        const int m = idx / nrows, r = idx % nrows, n = n0 + r;
        float v = res[m][r];
        if (ea.ss_in) v *= rinv[m];
        switch (epi) {
            case Epi::StoreF32:
                ea.out_f32[(long long)m * ea.ld_out + n] = v * ea.scale;
                break;
            case Epi::ResidAdd: {
                float* o = ea.out_f32 + (long long)m * ea.ld_out + n;
                const float x = *o + v;
                *o = x;
                if (ea.norm_y) ea.norm_y[(long long)m * ea.ld_out + n] = __float2bfloat16_rn(x * ea.norm_g[n]);
                res[m][r] = x;                              // for the norm partials below
                break;
            }
            case Epi::SwiGLU:                               // rows 2j = gate_j, 2j+1 = up_j
                if (!(n & 1)) {
                    const float u = res[m][r + 1] * (ea.ss_in ? rinv[m] : 1.f);
                    reinterpret_cast<bf16*>(ea.out_t)[(long long)m * ea.ld_out + n / 2] = __float2bfloat16_rn(siluf_(v) * u);
                }
                break;
            case Epi::Merge:                                // rows 2j = gate pre-activation, 2j+1 = feedback
                break;
            case Epi::LsePart:                              // not produced by this kernel
                break;
        }
    }
    if (epi == Epi::Merge) {
        // one thread per output column c: both rows of its pair are read before any is rewritten
        __syncthreads();
        const int ncols = nrows / 2;
        for (int idx = threadIdx.x; idx < M * ncols; idx += blockDim.x) {
            const int m = idx / ncols, j = idx % ncols, c = n0 / 2 + j;
            const float s = ea.ss_in ? rinv[m] : 1.f;
            const float g = res[m][2 * j] * s, u = res[m][2 * j + 1] * s;
            const bf16* e = reinterpret_cast<const bf16*>(ea.merge_e);
            const float x = __bfloat162float(e[(long long)m * ea.ld_e + c]) + sigmoidf_(g + ea.bias[c]) * u;
            ea.out_f32[(long long)m * ea.ld_out + c] = x;
            if (ea.norm_y) ea.norm_y[(long long)m * ea.ld_out + c] = __float2bfloat16_rn(x * ea.norm_g[c]);
            res[m][2 * j] = x;                             // the pair's first slot holds x for the partials
        }
    }
    if (ea.norm_y && (epi == Epi::ResidAdd || epi == Epi::Merge)) {
        // deferred-norm partials: sum of x^2 over each group of 16 output columns, fixed order
        __syncthreads();
        const int step = epi == Epi::Merge ? 2 : 1;         // GEMM rows per output column
        const int ngroups = nrows / (16 * step);
        for (int idx = threadIdx.x; idx < M * ngroups; idx += blockDim.x) {
            const int m = idx / ngroups, g = idx % ngroups;
            float ss = 0.f;
            for (int j = 0; j < 16; ++j) {
                const float x = res[m][(g * 16 + j) * step];
                ss += x * x;
            }
            ea.ss_out[(long long)m * ea.ss_ld + (n0 / step) / 16 + g] = ss;
        }
    }
}

int gv_rows_per_cta(int N) {
    // whole 32-row blocks, as many CTAs as fit two per SM, at most GV_MAX_ROWS rows each
    const int blocks = (N + 31) / 32;
    const int ctas_cap = 2 * sm_count();
    int per = (blocks + ctas_cap - 1) / ctas_cap;
    return per * 32;
}

template <int MB>
cudaError_t run_gemv(Launch L, Epi epi, const bf16* A, int lda, const bf16* W, int M, int N, int K, const EpiArgs& ea,
                     DevHeader* hdr) {
    const int rows = gv_rows_per_cta(N);
    const size_t chunk = (size_t)GV_WARPS * K * 2;
    const int stages = (int)min((size_t)GV_MAX_STAGES, (size_t)GV_RING_BYTES / chunk);
    const size_t smem = (size_t)stages * chunk + 128;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(k_gemv<MB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             GV_RING_BYTES + 128);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const unsigned grid = (unsigned)((N + rows - 1) / rows);
    return launch_k(L, k_gemv<MB>, grid, GV_WARPS * 32, smem, W, A, lda, M, N, K, rows, stages, epi, ea, hdr);
}

}  // namespace

bool gemv_shape_supported(int M, int N, int K, int lda) {
    // whole 32-row blocks per CTA, 16-byte pieces of every row, rows small enough for a ring of
    // at least two chunks
    if (M < 1 || M > 4 || N < 1 || N % 32 || K < 8 || K % 8 || lda % 8) return false;
    if ((size_t)GV_WARPS * K * 2 * 2 > (size_t)GV_RING_BYTES) return false;
    return gv_rows_per_cta(N) <= GV_MAX_ROWS;
}

// Measured on B200 against the few-row tensor-core kernel (single launches, weights from HBM):
// faster where the weight matrix gives every SM at least one 32-row block and rows are short
// (1 x 32768 x 2048: 37 vs 52 us; 1 x 8192 x 1024: 8.9 vs 10.2; 1 x 6144 x 2048: 10.9 vs 11.8),
// slower where a few dozen CTAs each stream long rows (1 x 2048 x 2048: 9.7 vs 5.4;
// 1 x 2048 x 5632: 18.5 vs 9.6; 4 x 2048 x 2048: 21.5 vs 5.5).
bool gemv_preferred(int M, int N, int K) {
    return gemv_shape_supported(M, N, K, K) && N >= 32 * sm_count() && K <= 2048;
}

bool gemv_supported(int M, int N, int K, int lda, const void* A, const void* W) {
    return gemv_shape_supported(M, N, K, lda) && reinterpret_cast<uintptr_t>(A) % 16 == 0 &&
           reinterpret_cast<uintptr_t>(W) % 16 == 0;
}

cudaError_t launch_gemv(Launch L, Epi epi, const bf16* A, int lda, const bf16* W, int M, int N, int K,
                        const EpiArgs& ea, DevHeader* hdr) {
    if (M == 1) return run_gemv<1>(L, epi, A, lda, W, M, N, K, ea, hdr);
    if (M == 2) return run_gemv<2>(L, epi, A, lda, W, M, N, K, ea, hdr);
    if (M <= 4) return run_gemv<4>(L, epi, A, lda, W, M, N, K, ea, hdr);
    return cudaErrorInvalidValue;
}

}  // namespace rlt
