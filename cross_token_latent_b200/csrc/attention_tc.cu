// Encoder causal self-attention on the sm_100a tensor cores (bf16, head_dim 64 or 128).
//
// One CTA computes 128 queries of one (sequence, head) against the causal key range in tiles
// of 128 keys, flash-attention style, with every operand K-major in the 128-byte swizzle
// layout that TMA writes:
//   warp 8, lane 0  TMA producer: the Q tile once, then K and V^T tiles into two stages;
//   warp 9          allocates / frees the 512 TMEM columns; lane 0 issues the MMAs: S_j = Q K_j^T
//                   into one of two S buffers (TMEM columns [0, 128) and [128, 256)) as soon as
//                   K_j has landed and the buffer's previous tile has been read, so the next
//                   tile's scores are ready while the softmax of this one runs; then O += P_j V_j
//                   into TMEM columns [256, 256 + head_dim) once P_j is written;
//   warps 0-7       softmax, two warps per TMEM lane quadrant: warp w owns query row
//                   32 (w % 4) + lane and key columns [64 h, 64 h + 64) of each tile, h = w / 4.
//                   The two halves of a row post their partial maxima to shared memory (an
//                   mbarrier per quadrant, bounded waits) and both continue with the row's
//                   maximum: causal mask on the diagonal tile, exp2, P rounded to bf16 into
//                   shared memory (the row sum is taken over the rounded values, so P V / sum
//                   stays a convex combination), rescale of their half of O in TMEM when the
//                   maximum grows, and the epilogue O / sum -> bf16 over their half of head_dim.
// V is stored transposed per (sequence, head) ([head_dim][T_pad], keys contiguous) so that it
// is a K-major B operand like the others.  Every mbarrier wait is bounded.
#include <cudaTypedefs.h>

#include "kernels.cuh"
#include "sm100.cuh"

namespace rlt {

namespace {

constexpr int QT = 128;   // queries per CTA (UMMA M)
constexpr int KT = 128;   // keys per tile (UMMA N of S and K of P V)

template <int HD>
struct FaShape {
    static constexpr int ATOMS = HD / 64;                 // 64-element swizzle atoms along head_dim
    static constexpr int Q_BYTES = QT * HD * 2;
    static constexpr int K_BYTES = KT * HD * 2;
    static constexpr int V_BYTES = HD * KT * 2;           // V^T tile: HD rows x 128 keys
    static constexpr int P_BYTES = QT * KT * 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;         // 2 stages
    static constexpr int OFF_V = OFF_K + 2 * K_BYTES;     // 2 stages
    static constexpr int OFF_P = OFF_V + 2 * V_BYTES;
    static constexpr int OFF_RED = OFF_P + P_BYTES;       // row-max exchange [2][2 halves][128 rows]
    static constexpr int OFF_BAR = OFF_RED + 2 * 2 * QT * 4;
    static constexpr int SMEM = OFF_BAR + 256 + 1024;
    static constexpr int TMEM_COLS = 512;
    static constexpr uint32_t S_COL = 0, O_COL = 256;     // S double-buffered at 0 and 128
};

constexpr int FA_SOFTMAX_WARPS = 8;                        // two per TMEM lane quadrant
constexpr int FA_THREADS = (FA_SOFTMAX_WARPS + 2) * 32;    // + TMA producer + MMA issuer

// 2^x by the ex2.approx instruction (relative error ~2^-22; flushes denormals to zero).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <int HD>
__global__ void __launch_bounds__(FA_THREADS, 1)
k_enc_fa_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
            const __grid_constant__ CUtensorMap tmV, bf16* __restrict__ o, int B, int Tn, int H, float qscale,
            DevHeader* hdr) {
    using S = FaShape<HD>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* q_full = reinterpret_cast<uint64_t*>(smem + S::OFF_BAR);
    uint64_t* kv_full = q_full + 1;       // [2]
    uint64_t* kv_empty = kv_full + 2;     // [2]
    uint64_t* s_full = kv_empty + 2;      // [2] S buffer b holds S_j for j % 2 == b
    uint64_t* s_free = s_full + 2;        // [2] the softmax warps have read S buffer b
    uint64_t* p_full = s_free + 2;        // P_j written and O rescaled
    uint64_t* o_done = p_full + 1;        // O += P_j V_j complete
    uint64_t* red_ready = o_done + 1;     // [2][4] both halves of a quadrant posted their row max
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(red_ready + 8);
    float* red = reinterpret_cast<float*>(smem + S::OFF_RED);
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_qt = (Tn + QT - 1) / QT;
    const int qt = n_qt - 1 - (int)blockIdx.x;            // longest causal ranges first
    const int bh = blockIdx.y;
    const int q0 = qt * QT;
    const int nt = qt + 1;                                 // key tiles 0..qt
    const int PRODUCER = FA_SOFTMAX_WARPS, ISSUER = FA_SOFTMAX_WARPS + 1;
    pdl_trigger();

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
            mbar_init(&s_full[s], 1);
            mbar_init(&s_free[s], FA_SOFTMAX_WARPS);
        }
        mbar_init(p_full, FA_SOFTMAX_WARPS);
        mbar_init(o_done, 1);
        for (int i = 0; i < 8; ++i) mbar_init(&red_ready[i], 64);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == ISSUER) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(S::TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == PRODUCER) {
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(&tmQ) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(&tmK) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(&tmV) : "memory");
            pdl_wait();
            mbar_expect_tx(q_full, S::Q_BYTES);
#pragma unroll
            for (int a = 0; a < S::ATOMS; ++a) tma_load_3d(smem + S::OFF_Q + a * QT * 128, &tmQ, q_full, 64 * a, q0, bh);
            for (int j = 0; j < nt; ++j) {
                int s = j & 1;
                uint32_t ph = (j >> 1) & 1;
                if (!mbar_wait(&kv_empty[s], ph ^ 1, &abort_flag)) { abort_flag = 1; break; }
                mbar_expect_tx(&kv_full[s], S::K_BYTES + S::V_BYTES);
                uint8_t* kb = smem + S::OFF_K + s * S::K_BYTES;
                uint8_t* vb = smem + S::OFF_V + s * S::V_BYTES;
#pragma unroll
                for (int a = 0; a < S::ATOMS; ++a) tma_load_3d(kb + a * KT * 128, &tmK, &kv_full[s], 64 * a, j * KT, bh);
#pragma unroll
                for (int a = 0; a < 2; ++a) tma_load_3d(vb + a * HD * 128, &tmV, &kv_full[s], j * KT + 64 * a, 0, bh);
            }
        }
    } else if (warp == ISSUER) {
        if (lane == 0) {
            constexpr uint32_t id_s = idesc_bf16(QT, KT), id_o = idesc_bf16(QT, HD);
            const uint32_t tO = tmem + S::O_COL;
            // S_j = Q K_j^T into S buffer j % 2, once K_j has landed and the softmax warps have
            // read that buffer's previous tile j - 2
            auto issue_s = [&](int j) -> bool {
                const int s = j & 1;
                if (!mbar_wait(&kv_full[s], (j >> 1) & 1, &abort_flag)) return false;
                if (j >= 2 && !mbar_wait(&s_free[s], ((j - 2) >> 1) & 1, &abort_flag)) return false;
                tc_fence_after();
                const uint32_t tS = tmem + S::S_COL + s * KT;
#pragma unroll
                for (int a = 0; a < S::ATOMS; ++a) {
                    uint64_t dq = sdesc_sw128(smem + S::OFF_Q + a * QT * 128);
                    uint64_t dk = sdesc_sw128(smem + S::OFF_K + s * S::K_BYTES + a * KT * 128);
#pragma unroll
                    for (int k = 0; k < 4; ++k) umma(tS, dq + 2 * k, dk + 2 * k, id_s, (a | k) != 0);
                }
                umma_commit(&s_full[s]);
                return true;
            };
            bool ok = mbar_wait(q_full, 0, &abort_flag) && issue_s(0);
            for (int j = 0; ok && j < nt; ++j) {
                const int s = j & 1;
                // the next tile's scores first, so the softmax warps never wait for them
                if (j + 1 < nt && !issue_s(j + 1)) { ok = false; break; }
                if (!mbar_wait(p_full, j & 1, &abort_flag)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    uint64_t dp = sdesc_sw128(smem + S::OFF_P + a * QT * 128);
                    uint64_t dv = sdesc_sw128(smem + S::OFF_V + s * S::V_BYTES + a * HD * 128);
#pragma unroll
                    for (int k = 0; k < 4; ++k) umma(tO, dp + 2 * k, dv + 2 * k, id_o, (j | a | k) != 0);
                }
                umma_commit(&kv_empty[s]);
                umma_commit(o_done);
            }
            if (!ok) abort_flag = 1;
        }
    } else {
        // softmax warps: warp w owns query row r = 32 (w % 4) + lane (TMEM lane quadrant w % 4)
        // and key columns [64 h, 64 h + 64) of every tile, h = w / 4; the two halves of a row
        // exchange their partial maxima through shared memory on an mbarrier.
        const int qd = warp & 3, hf = warp >> 2;
        const int r = qd * 32 + lane;
        const int q = q0 + r;
        const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
        const uint32_t tO = tmem + S::O_COL + lane_off + hf * (HD / 2);
        uint8_t* P = smem + S::OFF_P + hf * QT * 128;       // this half's 64-key swizzle atom
        float m = -1e30f, l = 0.f;
        bool ok = true;
        for (int j = 0; j < nt; ++j) {
            const int sb = j & 1;
            ok = ok && mbar_wait(&s_full[sb], (j >> 1) & 1, &abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            float sv[64];
            const uint32_t tS = tmem + S::S_COL + sb * KT + lane_off + hf * 64;
            tmem_ld32(tS, sv);
            tmem_ld32(tS + 32, sv + 32);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_free[sb]);
            // the maximum is taken over the raw scores (qscale > 0), and exp2 of
            // qscale * s - max is one fused multiply-add and one ex2.approx per element: the
            // probabilities are rounded to bf16 right after, far coarser than ex2.approx's error
            const bool diag = (j == nt - 1);
            float rmx = -1e30f;
            if (diag) {
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    if (j * KT + hf * 64 + c > q) sv[c] = -1e30f;
                    rmx = fmaxf(rmx, sv[c]);
                }
            } else {
#pragma unroll
                for (int c = 0; c < 64; ++c) rmx = fmaxf(rmx, sv[c]);
            }
            float mx = fmaxf(m, rmx * qscale);
            // the row's maximum over both halves
            float* rb = red + (size_t)sb * 2 * QT;
            rb[hf * QT + r] = mx;
            mbar_arrive(&red_ready[sb * 4 + qd]);
            ok = mbar_wait(&red_ready[sb * 4 + qd], (j >> 1) & 1, &abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            mx = fmaxf(mx, rb[(1 - hf) * QT + r]);
            const float alpha = ex2_approx(m - mx);
            const float nmx = -mx;
            float rowsum = 0.f;
            // P_j overwrites P_{j-1}: wait until P_{j-1} V_{j-1} has completed (it also makes O
            // final for the rescale below)
            if (j > 0) {
                ok = mbar_wait(o_done, (j - 1) & 1, &abort_flag);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                tc_fence_after();
            }
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                float p8[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) p8[i] = ex2_approx(fmaf(sv[ch * 8 + i], qscale, nmx));
                const uint4 packed = Vec16<bf16>::pack(p8);          // rounded to bf16 once
                Vec16<bf16>::unpack(packed, p8);                      // the rounded values
#pragma unroll
                for (int i = 0; i < 8; ++i) rowsum += p8[i];
                uint8_t* dst = P + r * 128 + ((ch ^ (r & 7)) << 4);
                *reinterpret_cast<uint4*>(dst) = packed;
            }
            l = l * alpha + rowsum;
            if (j > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {     // warp-collective TMEM access
#pragma unroll 1
                for (int c = 0; c < HD / 2; c += 32) {
                    float ov[32];
                    tmem_ld32(tO + c, ov);
#pragma unroll
                    for (int i = 0; i < 32; ++i) ov[i] *= alpha;
                    tmem_st32(tO + c, ov);
                }
            }
            m = mx;
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        pdl_wait();
        if (ok) {
            ok = mbar_wait(o_done, (nt - 1) & 1, &abort_flag);
            ok = __all_sync(0xffffffffu, ok);
        }
        if (ok) {
            // the row sum over both halves (the same exchange, on the buffer of tile nt)
            const int sb = nt & 1;
            float* rb = red + (size_t)sb * 2 * QT;
            rb[hf * QT + r] = l;
            mbar_arrive(&red_ready[sb * 4 + qd]);
            ok = mbar_wait(&red_ready[sb * 4 + qd], (nt >> 1) & 1, &abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) l += rb[(1 - hf) * QT + r];
        }
        if (ok) {
            tc_fence_after();
            const float inv = 1.0f / l;
            const int b = bh / H, h = bh % H;
            bf16* orow = o + ((long long)b * Tn + q) * H * HD + h * HD + hf * (HD / 2);
#pragma unroll 1
            for (int c = 0; c < HD / 2; c += 32) {
                float ov[32];
                tmem_ld32(tO + c, ov);
#pragma unroll
                for (int i = 0; i < 32; ++i) ov[i] *= inv;
                if (q < Tn) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8) st16(orow + c + i, Vec16<bf16>::pack(ov + i));
                }
            }
        } else if (lane == 0) {
            abort_flag = 1;
            raise_flag(hdr, ERR_TIMEOUT);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == ISSUER) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(S::TMEM_COLS));
    }
}

// V^T planes: qkv float32 [B*T, 3d] (v at columns 2d + h*hd) -> vt [B][H][hd][Tp] bf16 via a
// shared-memory tile transpose (32 positions x hd columns per block).
template <int HD>
__global__ void __launch_bounds__(256) k_enc_vt(const float* __restrict__ qkv, bf16* __restrict__ vt, int B, int Tn,
                                                int H, int Tp) {
    __shared__ float tile[32][HD + 1];
    pdl_wait();
    pdl_trigger();
    const int p0 = blockIdx.x * 32, h = blockIdx.y, b = blockIdx.z;
    const int d = H * HD;
    for (int i = threadIdx.x; i < 32 * HD; i += blockDim.x) {
        int pr = i / HD, c = i % HD;
        int p = p0 + pr;
        tile[pr][c] = p < Tn ? qkv[((long long)b * Tn + p) * 3 * d + 2 * d + h * HD + c] : 0.f;
    }
    __syncthreads();
    bf16* base = vt + ((long long)b * H + h) * HD * Tp;
    for (int i = threadIdx.x; i < 32 * HD; i += blockDim.x) {
        int c = i / 32, pr = i % 32;
        int p = p0 + pr;
        if (p < Tp) base[(long long)c * Tp + p] = __float2bfloat16_rn(tile[pr][c]);
    }
}

template <int HD>
cudaError_t run_fa(Launch L, const bf16* q, const bf16* k, const bf16* vt, bf16* o, int B, int Tn, int H, int Tp,
                   DevHeader* hdr) {
    using S = FaShape<HD>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(k_enc_fa_tc<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const uint64_t BH = (uint64_t)B * H;
    CUtensorMap tq, tk, tv;
    uint64_t qdims[3] = {(uint64_t)HD, (uint64_t)Tn, BH};
    uint64_t qstr[2] = {(uint64_t)HD * 2, (uint64_t)Tn * HD * 2};
    uint32_t qbox[3] = {64, QT, 1};
    uint64_t vdims[3] = {(uint64_t)Tn, (uint64_t)HD, BH};
    uint64_t vstr[2] = {(uint64_t)Tp * 2, (uint64_t)HD * Tp * 2};
    uint32_t vbox[3] = {64, (uint32_t)HD, 1};
    if (!tma_map_bf16(&tq, q, 3, qdims, qstr, qbox) || !tma_map_bf16(&tk, k, 3, qdims, qstr, qbox) ||
        !tma_map_bf16(&tv, vt, 3, vdims, vstr, vbox))
        return cudaErrorInvalidValue;
    dim3 grid((Tn + QT - 1) / QT, (unsigned)BH);
    const float qscale = 1.4426950408889634f / sqrtf((float)HD);
    return launch_k(L, k_enc_fa_tc<HD>, grid, FA_THREADS, S::SMEM, tq, tk, tv, o, B, Tn, H, qscale, hdr);
}

}  // namespace

int enc_vt_pitch(int Tn) { return (Tn + 7) / 8 * 8; }

bool enc_attention_tc_supported(int hd) { return hd == 64 || hd == 128; }

cudaError_t launch_enc_vt(Launch L, const float* qkv, bf16* vt, int B, int Tn, int H, int hd) {
    dim3 grid((unsigned)((enc_vt_pitch(Tn) + 31) / 32), (unsigned)H, (unsigned)B);
    int Tp = enc_vt_pitch(Tn);
    if (hd == 64) return launch_k(L, k_enc_vt<64>, grid, 256, 0, qkv, vt, B, Tn, H, Tp);
    if (hd == 128) return launch_k(L, k_enc_vt<128>, grid, 256, 0, qkv, vt, B, Tn, H, Tp);
    return cudaErrorInvalidValue;
}

cudaError_t launch_enc_attention_tc(Launch L, const bf16* q, const bf16* k, const bf16* vt, bf16* o, int B, int Tn,
                                    int H, int hd, DevHeader* hdr) {
    int Tp = enc_vt_pitch(Tn);
    if (hd == 64) return run_fa<64>(L, q, k, vt, o, B, Tn, H, Tp, hdr);
    if (hd == 128) return run_fa<128>(L, q, k, vt, o, B, Tn, H, Tp, hdr);
    return cudaErrorInvalidValue;
}

}  // namespace rlt
