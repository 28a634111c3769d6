// CUDA-core GEMM with fused epilogues: C[M, N] = A[M, K] x W[N, K]^T, float32 accumulation.
// Serves the float32 model mode, where the tensor cores do not apply, and any shape the
// tensor-core path does not take.  64x64 tiles, 256 threads, 4x4 outputs per thread.
#include "kernels.cuh"

namespace rlt {

namespace {

constexpr int BM = 64, BN = 64, BK = 16;

template <typename T>
struct EpiOps {
    // v[0..3] are columns n..n+3 of row m; `cnt` of them are inside N.
    __device__ __forceinline__ static void apply(Epi epi, const EpiArgs& ea, int m, int n, int cnt,
                                                 const float* v) {
        switch (epi) {
            case Epi::StoreF32: {
                float* o = ea.out_f32 + (long long)m * ea.ld_out + n;
                for (int j = 0; j < cnt; ++j) o[j] = v[j] * ea.scale;
                break;
            }
            case Epi::ResidAdd: {
                float* o = ea.out_f32 + (long long)m * ea.ld_out + n;
                for (int j = 0; j < cnt; ++j) o[j] += v[j];
                break;
            }
            case Epi::SwiGLU: {     // interleaved rows: column 2j = gate_j, 2j+1 = up_j
                T* o = reinterpret_cast<T*>(ea.out_t) + (long long)m * ea.ld_out + n / 2;
                for (int j = 0; j + 1 < cnt; j += 2) o[j / 2] = from_f<T>(siluf_(v[j]) * v[j + 1]);
                break;
            }
            case Epi::Merge: {      // interleaved rows: 2j = gate pre-activation, 2j+1 = feedback
                const T* e = reinterpret_cast<const T*>(ea.merge_e) + (long long)m * ea.ld_e;
                float* o = ea.out_f32 + (long long)m * ea.ld_out;
                for (int j = 0; j + 1 < cnt; j += 2) {
                    int c = (n + j) / 2;
                    o[c] = to_f(e[c]) + sigmoidf_(v[j] + ea.bias[c]) * v[j + 1];
                }
                break;
            }
        }
    }
};

template <typename T>
__global__ void __launch_bounds__(256) k_gemm_simt(const T* __restrict__ A, int lda, const T* __restrict__ W,
                                                   int M, int N, int K, Epi epi, EpiArgs ea) {
    pdl_wait();
    pdl_trigger();
    __shared__ float As[BK][BM + 4];
    __shared__ float Ws[BK][BN + 4];
    int tid = threadIdx.x;
    int tx = tid & 15, ty = tid >> 4;
    int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    float acc[4][4] = {};
    int lr = tid >> 2, lk = (tid & 3) * 4;   // loader: row 0..63, k offset 0,4,8,12
    for (int k0 = 0; k0 < K; k0 += BK) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            int k = k0 + lk + i;
            int m = m0 + lr, n = n0 + lr;
            As[lk + i][lr] = (m < M && k < K) ? to_f(A[(long long)m * lda + k]) : 0.f;
            Ws[lk + i][lr] = (n < N && k < K) ? to_f(W[(long long)n * K + k]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            float a[4], w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j] = Ws[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
        }
        __syncthreads();
    }
    int n = n0 + tx * 4;
    if (n >= N) return;
    int cnt = min(4, N - n);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int m = m0 + ty * 4 + i;
        if (m < M) EpiOps<T>::apply(epi, ea, m, n, cnt, acc[i]);
    }
}

}  // namespace

template <typename T>
cudaError_t launch_gemm_simt(Launch L, Epi epi, const T* A, int lda, const T* W, int M, int N, int K,
                             const EpiArgs& ea) {
    dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM);
    return launch_k(L, k_gemm_simt<T>, grid, 256, 0, A, lda, W, M, N, K, epi, ea);
}

template <>
cudaError_t launch_gemm<float>(Launch L, Epi epi, const float* A, int lda, const float* W, int M, int N, int K,
                               const EpiArgs& ea) {
    if (ea.norm_y || ea.ss_in) return cudaErrorInvalidValue;    // deferred norms: tensor-core paths only
    return launch_gemm_simt<float>(L, epi, A, lda, W, M, N, K, ea);
}

template <>
cudaError_t launch_gemm<bf16>(Launch L, Epi epi, const bf16* A, int lda, const bf16* W, int M, int N, int K,
                              const EpiArgs& ea) {
    if (M <= L.gemv_max_rows && gemv_preferred(M, N, K) && gemv_supported(M, N, K, lda, A, W))
        return launch_gemv(L, epi, A, lda, W, M, N, K, ea, ea.hdr);
    if (gemm_tc_supported(A, lda, W, K)) {
        if (gemm_swap_preferred(M, N, K)) return launch_gemm_swap(L, epi, A, lda, W, M, N, K, ea, ea.hdr);
        return launch_gemm_tc(L, epi, A, lda, W, M, N, K, ea, ea.hdr);
    }
    if (ea.norm_y || ea.ss_in) return cudaErrorInvalidValue;    // deferred norms: tensor-core paths only
    return launch_gemm_simt<bf16>(L, epi, A, lda, W, M, N, K, ea);
}

template cudaError_t launch_gemm_simt<float>(Launch, Epi, const float*, int, const float*, int, int, int,
                                             const EpiArgs&);
template cudaError_t launch_gemm_simt<bf16>(Launch, Epi, const bf16*, int, const bf16*, int, int, int,
                                            const EpiArgs&);

}  // namespace rlt
