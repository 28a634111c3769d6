// Tensor-core GEMM for few rows (M <= 64), the decode shape of small batches:
// C[M, N] = A[M, K] x W[N, K]^T computed as C^T = W A^T, so that the weight rows sit on the
// MMA's M = 128 side and the batch rows on its N side (NB = 16, 32 or 64).  Every CTA then
// streams its own 128-row slab of W exactly once, and only the small activation panel is
// re-read by every CTA; the K dimension can be split over a cluster of up to 8 CTAs (partial
// slabs reduced in rank order through distributed shared memory, as in gemm_tc.cu).
//
// Roles as in gemm_tc.cu: warp 0 lane 0 issues TMA loads (weights before the programmatic
// launch dependency wait, activations after it), warp 1 lane 0 issues tcgen05.mma, warp 2 owns
// the TMEM allocation, all four warps run the epilogue.  In the epilogue thread r of the CTA
// owns output column (feature) f0 + r and holds the NB batch rows of that column; adjacent
// lanes hold the gate/up (or gate/feedback) pairs of the interleaved SwiGLU and merge weights.
#include <cudaTypedefs.h>

#include "kernels.cuh"
#include "sm100.cuh"

namespace rlt {

namespace {

constexpr int FM = 128;                      // weight rows (features) per CTA: UMMA M
constexpr int KB = 64;                       // k-block: one 128-byte swizzle row
constexpr int W_BYTES = FM * KB * 2;

// KA 64-wide k-atoms per pipeline stage: [KA weight atoms][KA activation atoms] (larger
// stages shorten the k-loop: a stage is delivered at a nearly fixed rate, see gemm_tc.cu).
template <int NB, int STAGES, int SPLIT, int KA = 1>
struct SwShape {
    static constexpr int X_BYTES = NB * KB * 2;          // one activation atom
    static constexpr int STAGE_BYTES = KA * (W_BYTES + X_BYTES);
    static constexpr int TMEM_COLS = NB < 32 ? 32 : NB;
    static constexpr int ROWS_PER_OWNER = FM / SPLIT;
    // the owner's partials, batch-column-major per source rank: [SPLIT][NB][ROWS_PER_OWNER]
    static constexpr int RECV_BYTES = SPLIT > 1 ? SPLIT * NB * ROWS_PER_OWNER * 4 : 0;
    static constexpr int SMEM = STAGES * STAGE_BYTES + RECV_BYTES + 1024 + 256;
};

// Transposed epilogue: v[j] is output (row mb + j, column n) for j = 0..15.  Every lane of the
// warp must call it (the pair epilogues exchange values between lanes n and n ^ 1, and the
// deferred-norm partials are reduced across lanes).  `store` says whether this lane writes.
// Deferred-norm groups: for ResidAdd the 16 output columns of a half-warp (lanes 0 / 16 write
// the partial), for Merge the 16 output columns of a whole warp (lane 0 writes).
__device__ __forceinline__ void epilogue16_t(Epi epi, const EpiArgs& ea, int n, bool store, int mb, int M,
                                             const float* v) {
    switch (epi) {
        case Epi::StoreF32:
#pragma unroll
            for (int j = 0; j < 16; ++j)
                if (store && mb + j < M) ea.out_f32[(long long)(mb + j) * ea.ld_out + n] = v[j] * ea.scale;
            break;
        case Epi::ResidAdd: {
            // all 16 residual loads first: with a runtime row pitch the compiler cannot tell a
            // store from the next row's load, and would otherwise wait out one round trip per row
            float x[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) x[j] = (store && mb + j < M) ? ea.out_f32[(long long)(mb + j) * ea.ld_out + n] : 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const long long m = mb + j;
                x[j] += v[j];
                if (store && m < M) {
                    ea.out_f32[m * ea.ld_out + n] = x[j];
                    if (ea.norm_y) ea.norm_y[m * ea.ld_out + n] = __float2bfloat16_rn(x[j] * ea.norm_g[n]);
                }
                if (ea.norm_y) {
                    float sq = (store && m < M) ? x[j] * x[j] : 0.f;
#pragma unroll
                    for (int o = 8; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
                    if (store && m < M && (n & 15) == 0) ea.ss_out[m * ea.ss_ld + n / 16] = sq;
                }
            }
            break;
        }
        case Epi::SwiGLU: {     // feature 2c = gate_c, 2c+1 = up_c
            bf16* o = reinterpret_cast<bf16*>(ea.out_t);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                float up = __shfl_xor_sync(0xffffffffu, v[j], 1);
                if (store && !(n & 1) && mb + j < M)
                    o[(long long)(mb + j) * ea.ld_out + n / 2] = __float2bfloat16_rn(siluf_(v[j]) * up);
            }
            break;
        }
        case Epi::Merge: {      // feature 2c = gate pre-activation, 2c+1 = feedback projection
            const bf16* e = reinterpret_cast<const bf16*>(ea.merge_e);
            const int c = n / 2;
            const bool lead = store && !(n & 1);
            const float bias = lead ? ea.bias[c] : 0.f;
            float ev[16];                       // loads first (see ResidAdd)
#pragma unroll
            for (int j = 0; j < 16; ++j) ev[j] = (lead && mb + j < M) ? __bfloat162float(e[(long long)(mb + j) * ea.ld_e + c]) : 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const long long m = mb + j;
                float u = __shfl_xor_sync(0xffffffffu, v[j], 1);
                float x = 0.f;
                if (lead && m < M) {
                    x = ev[j] + sigmoidf_(v[j] + bias) * u;
                    ea.out_f32[m * ea.ld_out + c] = x;
                    if (ea.norm_y) ea.norm_y[m * ea.ld_out + c] = __float2bfloat16_rn(x * ea.norm_g[c]);
                }
                if (ea.norm_y) {
                    float sq = x * x;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
                    if (store && m < M && (n & 31) == 0) ea.ss_out[m * ea.ss_ld + c / 16] = sq;
                }
            }
            break;
        }
        case Epi::LsePart:      // not produced by this kernel
            break;
    }
}

template <int NB, int STAGES, int SPLIT, int KA>
__global__ void __launch_bounds__(128, 1)
k_gemm_swap(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, int M, int N, int K,
            Epi epi, EpiArgs ea, DevHeader* hdr) {
    using S = SwShape<NB, STAGES, SPLIT, KA>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* recv = reinterpret_cast<float*>(smem + STAGES * S::STAGE_BYTES);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * S::STAGE_BYTES + S::RECV_BYTES);
    uint64_t* empty = full + STAGES;
    uint64_t* done = empty + STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    __shared__ int abort_flag;
    __shared__ float rinv_s[NB];        // deferred-norm row scales of this CTA's batch rows

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int f0 = blockIdx.x * FM, b0 = blockIdx.y * NB;
    const int nkb_all = (K + KB * KA - 1) / (KB * KA);          // stages of KA atoms
    const uint32_t rank = SPLIT > 1 ? cluster_rank() : 0;
    const int per = (nkb_all + SPLIT - 1) / SPLIT;
    const int kb0 = min(nkb_all, (int)rank * per);
    const int nkb = min(nkb_all, kb0 + per) - kb0;
    pdl_trigger();
    if constexpr (SPLIT > 1) cluster_arrive_relaxed();

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(S::TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const uint64_t lim = ea.wait_ns;
    int armed = 0;                     // producer: k-blocks whose loads have been issued
    if (warp == 0 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmW) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmX) : "memory");
        // every CTA reads the same activation k-blocks: rotate the start (as in gemm_tc.cu)
        const int rot = nkb > 0 ? (int)(blockIdx.x % (unsigned)nkb) : 0;
        // element offset of atom q of stage kb
        auto kx = [&](int kb, int q) { return ((kb0 + (kb + rot) % nkb) * KA + q) * KB; };
        // the bounded-wait self-test (ea.no_loads) issues nothing
        const int pre = ea.no_loads ? 0 : (nkb < STAGES ? nkb : STAGES);
        for (int kb = 0; kb < pre; ++kb) {
            mbar_expect_tx(&full[kb], S::STAGE_BYTES);
#pragma unroll
            for (int q = 0; q < KA; ++q)
                tma_load_2d(smem + kb * S::STAGE_BYTES + q * W_BYTES, &tmW, &full[kb], kx(kb, q), f0);
        }
        pdl_wait();
        for (int kb = 0; kb < pre; ++kb)
#pragma unroll
            for (int q = 0; q < KA; ++q)
                tma_load_2d(smem + kb * S::STAGE_BYTES + KA * W_BYTES + q * S::X_BYTES, &tmX, &full[kb], kx(kb, q), b0);
        armed = pre;
        for (int kb = pre; kb < nkb && !ea.no_loads; ++kb) {
            int s = kb % STAGES;
            uint32_t ph = (kb / STAGES) & 1;
            if (!mbar_wait(&empty[s], ph ^ 1, &abort_flag, lim)) { abort_flag = 1; break; }
            uint8_t* st = smem + s * S::STAGE_BYTES;
            mbar_expect_tx(&full[s], S::STAGE_BYTES);
#pragma unroll
            for (int q = 0; q < KA; ++q) {
                tma_load_2d(st + q * W_BYTES, &tmW, &full[s], kx(kb, q), f0);
                tma_load_2d(st + KA * W_BYTES + q * S::X_BYTES, &tmX, &full[s], kx(kb, q), b0);
            }
            armed = kb + 1;
        }
    } else if (warp == 1 && lane == 0) {
        // after a timeout the issuer stops but still commits `done` (see gemm_tc.cu)
        constexpr uint32_t idesc = idesc_bf16(FM, NB);
        for (int kb = 0; kb < nkb; ++kb) {
            int s = kb % STAGES;
            uint32_t ph = (kb / STAGES) & 1;
            if (!mbar_wait(&full[s], ph, &abort_flag, lim)) { abort_flag = 1; break; }
            tc_fence_after();
            uint8_t* st = smem + s * S::STAGE_BYTES;
#pragma unroll
            for (int q = 0; q < KA; ++q) {
                const uint64_t dw = sdesc_sw128(st + q * W_BYTES), dx = sdesc_sw128(st + KA * W_BYTES + q * S::X_BYTES);
#pragma unroll
                for (int k = 0; k < KB / 16; ++k) umma(tmem, dw + 2 * k, dx + 2 * k, idesc, (kb | q | k) != 0);
            }
            umma_commit(&empty[s]);
        }
        if (nkb > 0) umma_commit(done);
    }
    __syncwarp();
    pdl_wait();

    // epilogue: thread r owns feature f0 + r, TMEM columns are batch rows b0 .. b0 + NB - 1
    const int r = warp * 32 + lane;
    const int n = f0 + r;
    const bool n_ok = n < N;
    if (ea.ss_in) {
        // warps 2 and 3 have no main-loop role: they compute the row scales while the MMAs run
        const int i = threadIdx.x - 64;
        if (i >= 0 && i < NB) rinv_s[i] = b0 + i < M ? deferred_rinv(ea, b0 + i) : 0.f;
        asm volatile("bar.sync 1, 128;" ::: "memory");
    }
    auto scale = [&](int c, float* v) {
        if (ea.ss_in) {
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] *= rinv_s[c + j];
        }
    };
    bool ok = nkb == 0 ? true : mbar_wait(done, 0, nullptr, lim);
    ok = __syncthreads_and(ok) && abort_flag == 0;      // no partial accumulator is stored
    tc_fence_after();
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    if constexpr (SPLIT == 1) {
        if (ok) {
#pragma unroll 1
            for (int c = 0; c < NB; c += 16) {
                float v[16];
                tmem_ld16(lane_base + c, v);
                scale(c, v);
                epilogue16_t(epi, ea, n, n_ok, b0 + c, M, v);
            }
        }
    } else {
        const uint32_t owner = (uint32_t)(r / S::ROWS_PER_OWNER);
        const int r_local = r - (int)owner * S::ROWS_PER_OWNER;
        cluster_wait_acquire();                                  // every CTA of the cluster has started
        if (ok) {
#pragma unroll 1
            for (int c = 0; c < NB; c += 16) {
                float v[16];
                if (nkb > 0) {
                    tmem_ld16(lane_base + c, v);
                } else {
#pragma unroll
                    for (int j = 0; j < 16; ++j) v[j] = 0.f;
                }
                // for every batch column the band's consecutive features are contiguous
                dsmem_store16_strided(recv + ((size_t)rank * NB + c) * S::ROWS_PER_OWNER + r_local,
                                      S::ROWS_PER_OWNER, owner, v);
            }
        }
        cluster_arrive_release();
        cluster_wait_acquire();                                  // all partials have landed
        // every lane runs the epilogue (the pair epilogues shuffle across lanes); lanes outside
        // this CTA's band only predicate their stores off
        if (ok) {
            const bool mine = owner == rank;
#pragma unroll 1
            for (int c = 0; c < NB; c += 16) {
                float v[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = 0.f;
                for (int src = 0; src < SPLIT; ++src) {
                    const float* p = recv + ((size_t)src * NB + c) * S::ROWS_PER_OWNER + r_local;
#pragma unroll
                    for (int j = 0; j < 16; ++j) v[j] += p[j * S::ROWS_PER_OWNER];
                }
                scale(c, v);
                epilogue16_t(epi, ea, n, n_ok && mine, b0 + c, M, v);
            }
        }
    }
    if (!ok && threadIdx.x == 0) {
        raise_flag(hdr, ERR_TIMEOUT);
        // wait (bounded) for the loads this CTA still has in flight before it exits
        for (int kb = armed > STAGES ? armed - STAGES : 0; kb < armed; ++kb)
            mbar_wait(&full[kb % STAGES], (kb / STAGES) & 1, nullptr, lim);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(S::TMEM_COLS));
    }
}

bool map2d(CUtensorMap* map, const void* ptr, int rows, int cols, int ld, int box_rows) {
    uint64_t dims[2] = {(uint64_t)cols, (uint64_t)rows};
    uint64_t strides[1] = {(uint64_t)ld * 2};
    uint32_t box[2] = {(uint32_t)KB, (uint32_t)box_rows};
    return tma_map_bf16(map, ptr, 2, dims, strides, box);
}

template <int NB, int STAGES, int SPLIT, int KA>
cudaError_t run_swap(Launch L, Epi epi, const bf16* A, int lda, const bf16* W, int M, int N, int K, const EpiArgs& ea,
                     DevHeader* hdr) {
    using S = SwShape<NB, STAGES, SPLIT, KA>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(k_gemm_swap<NB, STAGES, SPLIT, KA>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    CUtensorMap tw, tx;
    if (!map2d(&tw, W, N, K, K, FM) || !map2d(&tx, A, M, K, lda, NB)) return cudaErrorInvalidValue;
    dim3 grid((N + FM - 1) / FM, (M + NB - 1) / NB, SPLIT);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = S::SMEM;
    cfg.stream = L.stream;
    cudaLaunchAttribute attr[2];
    int na = 0;
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = L.pdl ? 1 : 0;
    ++na;
    if (SPLIT > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = 1;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = SPLIT;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    *L.count += 1;
    return cudaLaunchKernelEx(&cfg, k_gemm_swap<NB, STAGES, SPLIT, KA>, tw, tx, M, N, K, epi, ea, hdr);
}

template <int NB>
cudaError_t run_swap_split(int split, Launch L, Epi epi, const bf16* A, int lda, const bf16* W, int M, int N, int K,
                           const EpiArgs& ea, DevHeader* hdr) {
    // one CTA per SM: as many stages of two k-atoms (measured faster than one at every few-row
    // decode shape, e.g. 32 x 2048 x 5632 split 4: 10.85 -> 9.53 us) as fit next to the split
    // partials (~200 KB)
    constexpr int ST = NB == 64 ? 4 : 5;
    switch (split) {
        case 1: return run_swap<NB, ST, 1, 2>(L, epi, A, lda, W, M, N, K, ea, hdr);
        case 2: return run_swap<NB, ST, 2, 2>(L, epi, A, lda, W, M, N, K, ea, hdr);
        case 4: return run_swap<NB, ST, 4, 2>(L, epi, A, lda, W, M, N, K, ea, hdr);
        case 8: return run_swap<NB, ST, 8, 2>(L, epi, A, lda, W, M, N, K, ea, hdr);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

bool gemm_swap_supported(int M) { return M >= 1 && M <= 64; }

namespace {
int swap_nb(int M) { return M <= 16 ? 16 : (M <= 32 ? 32 : 64); }
long long swap_base(int M, int N) {
    const int nb = swap_nb(M);
    return (long long)((N + FM - 1) / FM) * ((M + nb - 1) / nb);
}
}  // namespace

// Measured on B200 at decode sizes: with at most 32 rows the swapped kernel wins or ties on
// every projection shape; at 33..64 rows it wins only when the weight matrix alone fills a
// wave with 128-row tiles (N >= ~6K), while narrower outputs run faster on the row-tile kernel
// whose 64-wide tiles put twice as many CTAs in flight.  Below four k-blocks the narrow
// row tiles win as well.
bool gemm_swap_preferred(int M, int N, int K) {
    if (!gemm_swap_supported(M)) return false;
    if ((K + KB - 1) / KB < 4) return false;
    if (M <= 32) return true;
    const long long base = swap_base(M, N);
    return base >= 48 && base <= 148;
}

// Fill one wave of SMs with at least two k-blocks per rank.  Clusters of 8 are left out: at
// one CTA per SM not every GPC holds two of them, so a 128-CTA grid of 8-CTA clusters runs in
// two waves (measured 2.2x the time of the 4-way split).
int gemm_swap_auto_split(int M, int N, int K) {
    const long long base = swap_base(M, N);
    const int nkb = (K + KB - 1) / KB;
    int split = 1;
    for (int s : {2, 4})
        if (base * s <= 148 && nkb >= 2 * s) split = s;
    return split;
}

cudaError_t launch_gemm_swap(Launch L, Epi epi, const bf16* A, int lda, const bf16* W, int M, int N, int K,
                             const EpiArgs& ea, DevHeader* hdr, int split) {
    if (!gemm_swap_supported(M)) return cudaErrorInvalidValue;
    const int nb = swap_nb(M);
    if (ea.norm_y && split > 4) split = 4;      // a deferred-norm group must stay in one owner band
    if (split <= 0) split = gemm_swap_auto_split(M, N, K);
    if (nb == 16) return run_swap_split<16>(split, L, epi, A, lda, W, M, N, K, ea, hdr);
    if (nb == 32) return run_swap_split<32>(split, L, epi, A, lda, W, M, N, K, ea, hdr);
    return run_swap_split<64>(split, L, epi, A, lda, W, M, N, K, ea, hdr);
}

}  // namespace rlt
