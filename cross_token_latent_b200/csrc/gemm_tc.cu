// Tensor-core GEMM for sm_100a: C[M, N] = A[M, K] x W[N, K]^T with bf16 operands, float32
// accumulation in tensor memory (TMEM) and the fused epilogues of the RLT path.
//
// One CTA computes one 128 x BN output tile with 4 warps (8 for the wide unsplit tiles):
//   warp 0, lane 0  TMA producer: 2-D tiled loads (128-byte swizzle) of A and W k-blocks of
//                   64 elements (KA of them per stage) into a ring of STAGES shared-memory
//                   slots (mbarrier full[s]);
//   warp 1, lane 0  MMA issuer: four tcgen05.mma (M=128, N=BN, K=16) per k-block into the
//                   TMEM accumulator; tcgen05.commit frees the slot (empty[s]) and, after
//                   the last block, signals the epilogue (done);
//   warp 2          allocates / frees the TMEM columns;
//   all warps       epilogue: warp w reads TMEM lanes 32(w%4)..32(w%4)+31 (one output row per
//                   thread; with 8 warps, warps w and w+4 take one half of the columns each)
//                   with tcgen05.ld and applies the fused epilogue, staged through shared
//                   memory.
// The file also holds the CTA-pair (cta_group::2) and the persistent variants.
// No load uses multicast.  Every mbarrier wait is bounded by %globaltimer; on
// expiry the CTA raises ERR_TIMEOUT, stops issuing work, frees its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>
#include <unordered_map>

#include "kernels.cuh"
#include "sm100.cuh"

namespace rlt {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;                       // 64 bf16 = 128 bytes = one swizzle row
constexpr int A_BYTES = BM * BK * 2;         // 16 KB
// Fused epilogue on 16 consecutive columns n..n+15 of row m (cnt of them inside N).  With a
// deferred norm to produce (ea.norm_y, ResidAdd / Merge only) it also writes bf16(x * g) and
// returns the sum of squares of the new x values it wrote (0 otherwise).
__device__ __forceinline__ float epilogue16(Epi epi, const EpiArgs& ea, int m, int n, int cnt, const float* v) {
    float ss = 0.f;
    switch (epi) {
        case Epi::StoreF32: {
            float* o = ea.out_f32 + (long long)m * ea.ld_out + n;
            if (cnt == 16) {
#pragma unroll
                for (int j = 0; j < 16; j += 4)
                    *reinterpret_cast<float4*>(o + j) =
                        make_float4(v[j] * ea.scale, v[j + 1] * ea.scale, v[j + 2] * ea.scale, v[j + 3] * ea.scale);
            } else {
                for (int j = 0; j < cnt; ++j) o[j] = v[j] * ea.scale;
            }
            break;
        }
        case Epi::ResidAdd: {
            float* o = ea.out_f32 + (long long)m * ea.ld_out + n;
            if (cnt == 16) {
                float x[16];
#pragma unroll
                for (int j = 0; j < 16; j += 4) {
                    float4 q = *reinterpret_cast<float4*>(o + j);
                    q.x += v[j]; q.y += v[j + 1]; q.z += v[j + 2]; q.w += v[j + 3];
                    *reinterpret_cast<float4*>(o + j) = q;
                    x[j] = q.x; x[j + 1] = q.y; x[j + 2] = q.z; x[j + 3] = q.w;
                }
                if (ea.norm_y) {
                    float y[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        y[j] = x[j] * ea.norm_g[n + j];
                        ss += x[j] * x[j];
                    }
                    bf16* yo = ea.norm_y + (long long)m * ea.ld_out + n;
                    st16(yo, Vec16<bf16>::pack(y));
                    st16(yo + 8, Vec16<bf16>::pack(y + 8));
                }
            } else {
                for (int j = 0; j < cnt; ++j) {
                    float x = o[j] + v[j];
                    o[j] = x;
                    if (ea.norm_y) {
                        ea.norm_y[(long long)m * ea.ld_out + n + j] = __float2bfloat16_rn(x * ea.norm_g[n + j]);
                        ss += x * x;
                    }
                }
            }
            break;
        }
        case Epi::SwiGLU: {     // columns 2j = gate_j, 2j+1 = up_j
            bf16* o = reinterpret_cast<bf16*>(ea.out_t) + (long long)m * ea.ld_out + n / 2;
            if (cnt == 16) {
                float h[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) h[j] = siluf_(v[2 * j]) * v[2 * j + 1];
                st16(o, Vec16<bf16>::pack(h));
            } else {
                for (int j = 0; j + 1 < cnt; j += 2) o[j / 2] = __float2bfloat16_rn(siluf_(v[j]) * v[j + 1]);
            }
            break;
        }
        case Epi::Merge: {      // columns 2j = gate pre-activation, 2j+1 = feedback projection
            const bf16* e = reinterpret_cast<const bf16*>(ea.merge_e) + (long long)m * ea.ld_e;
            float* o = ea.out_f32 + (long long)m * ea.ld_out;
            if (cnt == 16) {
                // output columns c0 .. c0+7 (c0 a multiple of 8): vector loads of e and the bias
                // before any store
                const int c0 = n / 2;
                float ev[8], bv[8], x[8];
                Vec16<bf16>::unpack(ld16(e + c0), ev);
                Vec16<float>::unpack(ld16(ea.bias + c0), bv);
                Vec16<float>::unpack(ld16(ea.bias + c0 + 4), bv + 4);
#pragma unroll
                for (int j = 0; j < 8; ++j) x[j] = ev[j] + sigmoidf_(v[2 * j] + bv[j]) * v[2 * j + 1];
                st16(o + c0, Vec16<float>::pack(x));
                st16(o + c0 + 4, Vec16<float>::pack(x + 4));
                if (ea.norm_y) {
                    float y[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        y[j] = x[j] * ea.norm_g[c0 + j];
                        ss += x[j] * x[j];
                    }
                    st16(ea.norm_y + (long long)m * ea.ld_out + c0, Vec16<bf16>::pack(y));
                }
                break;
            }
            for (int j = 0; j + 1 < cnt; j += 2) {
                int c = (n + j) / 2;
                float x = __bfloat162float(e[c]) + sigmoidf_(v[j] + ea.bias[c]) * v[j + 1];
                o[c] = x;
                if (ea.norm_y) {
                    ea.norm_y[(long long)m * ea.ld_out + c] = __float2bfloat16_rn(x * ea.norm_g[c]);
                    ss += x * x;
                }
            }
            break;
        }
        case Epi::LsePart:      // handled by the kernel's own epilogue loop
            break;
    }
    return ss;
}

// Per-row bookkeeping of a deferred norm around the 16-column epilogue chunks of one row:
// the consumer's row scale, and the producer's group partial sums (16 output columns per
// group = 16 GEMM columns, or 32 for the interleaved merge).  Tiles start on multiples of 32
// columns, so a group never straddles two tiles.
struct RowNorm {
    float rinv = 1.f;
    float acc = 0.f;
    __device__ __forceinline__ void scale(const EpiArgs& ea, float* v) const {
        if (ea.ss_in) {
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] *= rinv;
        }
    }
    __device__ __forceinline__ void scale32(const EpiArgs& ea, float* v) const {
        if (ea.ss_in) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] *= rinv;
        }
    }
    __device__ __forceinline__ void add(Epi epi, const EpiArgs& ea, int m, int n, int N, float part) {
        if (!ea.norm_y) return;
        acc += part;
        const int gw = epi == Epi::Merge ? 32 : 16;
        if ((n + 16) % gw == 0 || n + 16 >= N) {
            ea.ss_out[(long long)m * ea.ss_ld + n / gw] = acc;
            acc = 0.f;
        }
    }
};

// Fused head (Epi::LsePart): nothing is stored per logit.  For row m, lse_partial returns the
// (max, sum of exp) of z = acc * scale over accumulator columns c_begin .. c_end - 1 of the tile
// (those below N), and the thread whose columns hold the row's target writes its z to z_tok[m];
// the tile's (max, sum) goes to lse_part[m * lse_ld + tn].  The exponentials use ex2.approx
// (relative error near 2^-22): the log-sum-exp and the log-probs are outputs only, nothing of
// the recurrent state depends on them.  Warp-collective (TMEM loads).
constexpr float LOG2E_F = 1.4426950408889634f;
__device__ __forceinline__ float exp_fast(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x * LOG2E_F));
    return y;
}
template <int BN>
__device__ __forceinline__ float2 lse_partial(const EpiArgs& ea, uint32_t lane_base, int m, int M, int n0, int N,
                                              int c_begin, int c_end) {
    int tk = -1;
    if (m < M && ea.lse_tok) {
        tk = ea.lse_tok[(long long)m * ea.tok_stride];
        if (tk < 0 || tk >= N) tk = 0;
    }
    float mx = -INFINITY, sm = 0.f;
#pragma unroll 1
    for (int c = c_begin; c < c_end; c += 16) {
        float v[16];
        tmem_ld16(lane_base + c, v);
        const int n = n0 + c;
        if (m < M && n < N) {
            const int cnt = min(16, N - n);
            float cm = -INFINITY;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                v[j] *= ea.scale;
                if (j < cnt) cm = fmaxf(cm, v[j]);
                if (n + j == tk) ea.z_tok[m] = v[j];
            }
            if (cm > mx) {
                sm *= exp_fast(mx - cm);
                mx = cm;
            }
#pragma unroll
            for (int j = 0; j < 16; ++j)
                if (j < cnt) sm += exp_fast(v[j] - mx);
        }
    }
    return make_float2(mx, sm);
}
// (max, sum of exp) of two column ranges, a's first
__device__ __forceinline__ float2 lse_merge(float2 a, float2 b) {
    const float mx = fmaxf(a.x, b.x);
    if (mx == -INFINITY) return make_float2(mx, 0.f);
    return make_float2(mx, a.y * exp_fast(a.x - mx) + b.y * exp_fast(b.x - mx));
}
template <int BN>
__device__ __forceinline__ void lse_row(const EpiArgs& ea, uint32_t lane_base, int m, int M, int n0, int N, int tn) {
    const float2 p = lse_partial<BN>(ea, lane_base, m, M, n0, N, 0, BN);
    if (m < M) ea.lse_part[(long long)m * ea.lse_ld + tn] = p;
}
// AND of v over the nthreads threads that meet at named barrier id (all of them must arrive).
__device__ __forceinline__ bool bar_and(int id, int nthreads, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// ---- Staged epilogue.  A warp owns 32 consecutive output rows (lane = row).  Writing each
// row's values with its own thread puts the 32 lanes of every store on 32 different rows, i.e.
// 32 separate memory transactions per instruction; the staged path instead passes 32-column
// chunks through the warp's 4 KB staging area in shared memory (32 rows x 128 bytes, 16-byte
// pieces XOR-swizzled by row, so that both the row-wise and the column-wise accesses are free of
// bank conflicts) and moves whole row segments: every global instruction of the warp then
// covers 4 rows x 128 bytes (or 8 x 64, 16 x 32).  The arithmetic per element is that of
// epilogue16, in the same order.
constexpr int STG_BYTES = 32 * 128;          // one warp's staging area

__device__ __forceinline__ uint4* stg_at(uint8_t* stg, int row, int piece) {
    return reinterpret_cast<uint4*>(stg + row * 128 + ((piece ^ (row & 7)) << 4));
}
// rows row0 .. row0+31 (those below M) of `row_bytes` (32, 64 or 128) bytes each, between the
// staging area and global memory at g + (row0 + r) * ld_bytes
template <int ROW_BYTES>
__device__ __forceinline__ void stg_store_rows(uint8_t* stg, uint8_t* g, long long ld_bytes, int row0, int M) {
    constexpr int PPR = ROW_BYTES / 16, RPI = 32 / PPR;      // pieces per row, rows per instruction
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int i = 0; i < PPR; ++i) {
        const int r = i * RPI + lane / PPR, pc = lane % PPR;
        if (row0 + r < M) st16(g + (row0 + r) * ld_bytes + pc * 16, *stg_at(stg, r, pc));
    }
}
template <int ROW_BYTES>
__device__ __forceinline__ void stg_load_rows(uint8_t* stg, const uint8_t* g, long long ld_bytes, int row0, int M) {
    constexpr int PPR = ROW_BYTES / 16, RPI = 32 / PPR;
    const int lane = threadIdx.x & 31;
    uint4 t[PPR];
#pragma unroll
    for (int i = 0; i < PPR; ++i) {
        const int r = i * RPI + lane / PPR, pc = lane % PPR;
        t[i] = row0 + r < M ? ld16(g + (row0 + r) * ld_bytes + pc * 16) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < PPR; ++i) *stg_at(stg, i * RPI + lane / PPR, lane % PPR) = t[i];
}

// Whether the 32 columns n .. n+31 can take the staged path: the chunk lies inside N and every
// row segment it moves starts on a 16-byte boundary.
__device__ __forceinline__ bool staged_ok(Epi epi, const EpiArgs& ea, int n, int N) {
    if (n + 32 > N) return false;
    switch (epi) {
        case Epi::StoreF32:
            return ((reinterpret_cast<uintptr_t>(ea.out_f32) | ((uintptr_t)ea.ld_out * 4)) & 15) == 0;
        case Epi::ResidAdd:
            return ((reinterpret_cast<uintptr_t>(ea.out_f32) | ((uintptr_t)ea.ld_out * 4)) & 15) == 0 &&
                   (!ea.norm_y || (reinterpret_cast<uintptr_t>(ea.norm_y) & 15) == 0);
        case Epi::SwiGLU:
            return ((reinterpret_cast<uintptr_t>(ea.out_t) | ((uintptr_t)ea.ld_out * 2)) & 15) == 0;
        default:
            return false;
    }
}

// The staged epilogue of columns n .. n+31 for rows row0 .. row0+31 (this lane: row0 + lane),
// v = this lane's 32 accumulators after the deferred norm's scale.  Warp-collective.
__device__ __forceinline__ void epilogue32_staged(Epi epi, const EpiArgs& ea, int row0, int M, int n, float* v,
                                                  uint8_t* stg) {
    const int lane = threadIdx.x & 31, m = row0 + lane;
    switch (epi) {
        case Epi::StoreF32: {
#pragma unroll
            for (int p = 0; p < 8; ++p)
                *stg_at(stg, lane, p) = make_uint4(__float_as_uint(v[4 * p] * ea.scale), __float_as_uint(v[4 * p + 1] * ea.scale),
                                                   __float_as_uint(v[4 * p + 2] * ea.scale),
                                                   __float_as_uint(v[4 * p + 3] * ea.scale));
            __syncwarp();
            stg_store_rows<128>(stg, reinterpret_cast<uint8_t*>(ea.out_f32 + n), (long long)ea.ld_out * 4, row0, M);
            __syncwarp();
            break;
        }
        case Epi::ResidAdd: {
            uint8_t* xg = reinterpret_cast<uint8_t*>(ea.out_f32 + n);
            const long long xld = (long long)ea.ld_out * 4;
            stg_load_rows<128>(stg, xg, xld, row0, M);
            __syncwarp();
            float x[32];
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                float t[4];
                Vec16<float>::unpack(*stg_at(stg, lane, p), t);
#pragma unroll
                for (int j = 0; j < 4; ++j) x[4 * p + j] = t[j] + v[4 * p + j];
            }
            __syncwarp();
#pragma unroll
            for (int p = 0; p < 8; ++p) *stg_at(stg, lane, p) = Vec16<float>::pack(x + 4 * p);
            __syncwarp();
            stg_store_rows<128>(stg, xg, xld, row0, M);
            if (ea.norm_y) {
                float y[32];
                float ss0 = 0.f, ss1 = 0.f;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    y[j] = x[j] * ea.norm_g[n + j];
                    ss0 += x[j] * x[j];
                }
#pragma unroll
                for (int j = 16; j < 32; ++j) {
                    y[j] = x[j] * ea.norm_g[n + j];
                    ss1 += x[j] * x[j];
                }
                __syncwarp();
#pragma unroll
                for (int p = 0; p < 4; ++p) *stg_at(stg, lane, p) = Vec16<bf16>::pack(y + 8 * p);
                __syncwarp();
                stg_store_rows<64>(stg, reinterpret_cast<uint8_t*>(ea.norm_y + n), (long long)ea.ld_out * 2, row0, M);
                if (m < M) {
                    ea.ss_out[(long long)m * ea.ss_ld + n / 16] = ss0;
                    ea.ss_out[(long long)m * ea.ss_ld + n / 16 + 1] = ss1;
                }
            }
            __syncwarp();
            break;
        }
        case Epi::SwiGLU: {     // columns 2j = gate_j, 2j+1 = up_j -> 16 outputs at n / 2
            float h[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) h[j] = siluf_(v[2 * j]) * v[2 * j + 1];
            *stg_at(stg, lane, 0) = Vec16<bf16>::pack(h);
            *stg_at(stg, lane, 1) = Vec16<bf16>::pack(h + 8);
            __syncwarp();
            stg_store_rows<32>(stg, reinterpret_cast<uint8_t*>(reinterpret_cast<bf16*>(ea.out_t) + n / 2),
                               (long long)ea.ld_out * 2, row0, M);
            __syncwarp();
            break;
        }
        default:
            break;
    }
}

// The epilogue of one accumulator row m (TMEM lanes at lane_base, columns n0 + c_begin ..
// n0 + c_end - 1 of output column tile tn; LsePart takes all BN columns), through the warp's
// staging area stg where the chunk allows it.  Warp-collective (TMEM loads, staging).
template <int BN>
__device__ __forceinline__ void epilogue_row(Epi epi, const EpiArgs& ea, uint32_t lane_base, int m, int M, int n0,
                                             int N, int tn, RowNorm& rn, uint8_t* stg, int c_begin = 0,
                                             int c_end = BN) {
    if (epi == Epi::LsePart) {
        lse_row<BN>(ea, lane_base, m, M, n0, N, tn);
        return;
    }
    const int row0 = m - (int)(threadIdx.x & 31);
#pragma unroll 1
    for (int c = c_begin; c < c_end; c += 32) {
        const int n = n0 + c;
        if (staged_ok(epi, ea, n, N)) {
            float v[32];
            tmem_ld32(lane_base + c, v);
            rn.scale32(ea, v);
            epilogue32_staged(epi, ea, row0, M, n, v, stg);
            continue;
        }
#pragma unroll 1
        for (int h = c; h < c + 32 && h < c_end; h += 16) {
            float v[16];
            tmem_ld16(lane_base + h, v);
            if (m < M && n0 + h < N) {
                rn.scale(ea, v);
                rn.add(epi, ea, m, n0 + h, N, epilogue16(epi, ea, m, n0 + h, min(16, N - n0 - h), v));
            }
        }
    }
}

// KA: 64-wide k-atoms per pipeline stage.  A stage of narrow tiles is delivered at a roughly
// fixed rate per stage (measured on B200 at decode sizes: ~0.29 us per 64-wide stage for 32-,
// 64- and 128-column tiles with 4 to 10 stages in flight, ~0.43 us per 128-wide stage), so
// two atoms per stage shorten the k-loop of the narrow tiles by about a quarter.  A stage is
// [KA atoms of A (16 KB each)][KA atoms of W].
template <int BN, int STAGES, int SPLIT, int KA = 1>
struct TcShape {
    static constexpr int B_BYTES = BN * BK * 2;                // one W atom
    static constexpr int STAGE_BYTES = KA * (A_BYTES + B_BYTES);
    static constexpr int TMEM_COLS = BN < 32 ? 32 : BN;
    // split-K: the owner CTA of a row band receives every rank's partial rows here
    static constexpr int BAND = BN / SPLIT;          // split-K: output columns each rank owns
    // the owner's partials, column-major per source rank: [SPLIT][BAND][BM] floats
    static constexpr int RECV_BYTES = SPLIT > 1 ? SPLIT * BAND * BM * 4 : 0;
    static_assert(SPLIT == 1 || BAND % 16 == 0, "column bands are whole 16-column chunks");
    static constexpr int SMEM = STAGES * STAGE_BYTES + RECV_BYTES + 1024 + 256;
};

// SPLIT > 1: the grid's z dimension splits the k-blocks over a cluster of SPLIT CTAs that
// compute the same output tile.  Each CTA accumulates its share in its own TMEM, then sends
// each column band of its partial tile (BN / SPLIT columns per rank) to the CTA that owns the
// band through distributed shared memory; the owner adds the SPLIT partials in rank order (the
// same order for every element and every run) and applies the epilogue with all 128 threads.
// EW = 8 (wide tiles without a split): four more warps join the epilogue only, warps w and w + 4
// sharing TMEM lane quadrant w and taking one half of the tile's columns each.
template <int BN, int STAGES, int SPLIT, int KA, int EW>
__global__ void __launch_bounds__(EW * 32, 1)
k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW, int M, int N, int K,
          Epi epi, EpiArgs ea, DevHeader* hdr) {
    using S = TcShape<BN, STAGES, SPLIT, KA>;
    static_assert(EW == 4 || (EW == 8 && SPLIT == 1 && BN >= 64), "eight epilogue warps: unsplit tiles");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* recv = reinterpret_cast<float*>(smem + STAGES * S::STAGE_BYTES);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * S::STAGE_BYTES + S::RECV_BYTES);
    uint64_t* empty = full + STAGES;
    uint64_t* done = empty + STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    const int nkb_all = (K + BK * KA - 1) / (BK * KA);          // stages of KA atoms
    const uint32_t rank = SPLIT > 1 ? cluster_rank() : 0;
    const int per = (nkb_all + SPLIT - 1) / SPLIT;
    const int kb0 = min(nkb_all, (int)rank * per);
    const int nkb = min(nkb_all, kb0 + per) - kb0;
    pdl_trigger();
    if constexpr (SPLIT > 1) cluster_arrive_relaxed();     // peers may write here once all have started

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
        // TMA producer.  Weight tiles do not depend on the previous kernel: the first stages'
        // W loads are issued before the programmatic-launch dependency wait, the activation
        // (A) loads after it.  The bounded-wait self-test (ea.no_loads) issues nothing.
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmA) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmW) : "memory");
        const int pre = ea.no_loads ? 0 : (nkb < STAGES ? nkb : STAGES);
        for (int kb = 0; kb < pre; ++kb) {
            uint8_t* a = smem + kb * S::STAGE_BYTES;
            mbar_expect_tx(&full[kb], S::STAGE_BYTES);
#pragma unroll
            for (int q = 0; q < KA; ++q)
                tma_load_2d(a + KA * A_BYTES + q * S::B_BYTES, &tmW, &full[kb], ((kb0 + kb) * KA + q) * BK, n0);
        }
        pdl_wait();
        for (int kb = 0; kb < pre; ++kb)
#pragma unroll
            for (int q = 0; q < KA; ++q)
                tma_load_2d(smem + kb * S::STAGE_BYTES + q * A_BYTES, &tmA, &full[kb], ((kb0 + kb) * KA + q) * BK, m0);
        armed = pre;
        for (int kb = pre; kb < nkb && !ea.no_loads; ++kb) {
            int s = kb % STAGES;
            uint32_t ph = (kb / STAGES) & 1;
            if (!mbar_wait(&empty[s], ph ^ 1, &abort_flag, lim)) { abort_flag = 1; break; }
            uint8_t* a = smem + s * S::STAGE_BYTES;
            mbar_expect_tx(&full[s], S::STAGE_BYTES);
#pragma unroll
            for (int q = 0; q < KA; ++q) {
                tma_load_2d(a + q * A_BYTES, &tmA, &full[s], ((kb0 + kb) * KA + q) * BK, m0);
                tma_load_2d(a + KA * A_BYTES + q * S::B_BYTES, &tmW, &full[s], ((kb0 + kb) * KA + q) * BK, n0);
            }
            armed = kb + 1;
        }
    } else if (warp == 1 && lane == 0) {
        // MMA issuer.  After a timeout it stops issuing but still commits `done`, which then
        // tracks the MMAs already issued, so that none is in flight when TMEM is freed.
        constexpr uint32_t idesc = idesc_bf16(BM, BN);
        for (int kb = 0; kb < nkb; ++kb) {
            int s = kb % STAGES;
            uint32_t ph = (kb / STAGES) & 1;
            if (!mbar_wait(&full[s], ph, &abort_flag, lim)) { abort_flag = 1; break; }
            tc_fence_after();
            uint8_t* a = smem + s * S::STAGE_BYTES;
#pragma unroll
            for (int q = 0; q < KA; ++q) {
                const uint64_t da = sdesc_sw128(a + q * A_BYTES), dw = sdesc_sw128(a + KA * A_BYTES + q * S::B_BYTES);
#pragma unroll
                for (int k = 0; k < BK / 16; ++k)  // advance 16 elements = 32 bytes = 2 in (addr >> 4)
                    umma(tmem, da + 2 * k, dw + 2 * k, idesc, (kb | q | k) != 0);
            }
            umma_commit(&empty[s]);
        }
        if (nkb > 0) umma_commit(done);
    }
    __syncwarp();
    pdl_wait();

    // epilogue: thread owns output row m0 + 32 * (warp % 4) + lane (a split rank with no
    // k-blocks has issued no MMA and contributes zeros)
    const int qd = warp & 3, chalf = EW == 8 ? warp >> 2 : 0;
    RowNorm rn;
    if (ea.ss_in && m0 + qd * 32 + lane < M) rn.rinv = deferred_rinv(ea, m0 + qd * 32 + lane);
    bool ok = nkb == 0 ? true : mbar_wait(done, 0, nullptr, lim);
    // a producer or issuer that gave up raised abort_flag before this barrier: no thread then
    // stores a partial accumulator
    ok = __syncthreads_and(ok) && abort_flag == 0;
    tc_fence_after();
    const uint32_t lane_base = tmem + ((uint32_t)(qd * 32) << 16);
    if constexpr (SPLIT == 1) {
        // every stage of the ring has been consumed: its first EW * 4 KB are the warps' staging
        // areas.  With eight warps each half of the columns has its own warp (the fused head's
        // per-row reduction stays with the first four).
        if (ok && EW == 8 && epi == Epi::LsePart) {
            // each half reduces its columns; the second half's (max, sum) pass through shared
            // memory (past the staging areas) to the first, which merges them in column order
            const int m = m0 + qd * 32 + lane;
            const float2 part = lse_partial<BN>(ea, lane_base, m, M, n0, N, chalf * (BN / 2), (chalf + 1) * (BN / 2));
            float2* xbuf = reinterpret_cast<float2*>(smem + EW * STG_BYTES);
            if (chalf == 1) xbuf[qd * 32 + lane] = part;
            __syncthreads();
            if (chalf == 0 && m < M) ea.lse_part[(long long)m * ea.lse_ld + blockIdx.x] = lse_merge(part, xbuf[qd * 32 + lane]);
        } else if (ok && EW == 4) {
            epilogue_row<BN>(epi, ea, lane_base, m0 + qd * 32 + lane, M, n0, N, blockIdx.x, rn, smem + warp * STG_BYTES);
        } else if (ok) {
            epilogue_row<BN>(epi, ea, lane_base, m0 + qd * 32 + lane, M, n0, N, blockIdx.x, rn, smem + warp * STG_BYTES,
                             chalf * (BN / 2), (chalf + 1) * (BN / 2));
        }
    } else {
        // Column bands: rank r owns output columns [r * BAND, (r + 1) * BAND) of the tile for
        // all 128 rows, so every thread keeps its row.  It sends each band of its partial row
        // to that band's owner, column-major (for every column a warp's 32 rows are 128
        // contiguous bytes, so each remote store instruction is one coalesced transfer), then
        // adds the SPLIT partials of its own band in rank order (the same order for every
        // element and every run) and applies the epilogue.
        const int row = warp * 32 + lane;
        cluster_wait_acquire();                                  // every CTA of the cluster has started
        if (ok) {
#pragma unroll 1
            for (int c = 0; c < BN; c += 16) {
                float v[16];
                if (nkb > 0) {
                    tmem_ld16(lane_base + c, v);
                } else {
#pragma unroll
                    for (int j = 0; j < 16; ++j) v[j] = 0.f;
                }
                dsmem_store16_strided(recv + ((size_t)rank * S::BAND + c % S::BAND) * BM + row, BM,
                                      (uint32_t)(c / S::BAND), v);
            }
        }
        cluster_arrive_release();
        cluster_wait_acquire();                                  // all partials have landed
        if (ok) {
            const int m = m0 + row;
            uint8_t* stg = smem + warp * STG_BYTES;       // the consumed ring
#pragma unroll 1
            for (int c = 0; c < S::BAND; c += 16) {
                const int n = n0 + (int)rank * S::BAND + c;
                if (S::BAND % 32 == 0 && c % 32 == 0 && staged_ok(epi, ea, n, N)) {
                    float v[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = 0.f;
                    for (int src = 0; src < SPLIT; ++src) {
                        const float* p = recv + ((size_t)src * S::BAND + c) * BM + row;
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] += p[j * BM];
                    }
                    rn.scale32(ea, v);
                    epilogue32_staged(epi, ea, m0 + warp * 32, M, n, v, stg);
                    c += 16;                               // the chunk covered 32 columns
                    continue;
                }
                float v[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = 0.f;
                for (int src = 0; src < SPLIT; ++src) {
                    const float* p = recv + ((size_t)src * S::BAND + c) * BM + row;
#pragma unroll
                    for (int j = 0; j < 16; ++j) v[j] += p[j * BM];
                }
                if (m < M && n < N) {
                    rn.scale(ea, v);
                    rn.add(epi, ea, m, n, N, epilogue16(epi, ea, m, n, min(16, N - n), v));
                }
            }
        }
    }
    if (!ok) {
        if (threadIdx.x == 0) {
            raise_flag(hdr, ERR_TIMEOUT);
            // wait (bounded) for the loads this CTA still has in flight before it exits
            for (int kb = armed > STAGES ? armed - STAGES : 0; kb < armed; ++kb)
                mbar_wait(&full[kb % STAGES], (kb / STAGES) & 1, nullptr, lim);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(S::TMEM_COLS));
    }
}

// CTA-pair row-tile GEMM: a cluster of two CTAs computes one 256 x BN output tile with
// tcgen05.mma.cta_group::2 (M = 256).  CTA r of the pair stages rows 128 r .. 128 r + 127 of the
// A tile and rows (BN / 2) r .. (BN / 2)(r + 1) - 1 of the W tile, so each CTA reads 1/3 fewer
// bytes per k-block than a 128 x BN tile of the same MMA work, and holds accumulator rows 128 r ..
// in its own TMEM.  Roles per CTA as in k_gemm_tc, except:
//   - both producers' loads complete on the leader's (rank 0) full[s] barrier, which the leader
//     arms for both CTAs' bytes (a load landing first leaves the barrier's transaction count
//     below zero until the leader arrives, so the phase cannot complete early);
//   - the leader's lane issues the pair MMAs; its commits arrive on empty[s] and done in both
//     CTAs, so each producer refills its own stage and each CTA's epilogue starts on its own;
//     after a timeout the leader commits to its own `drain` barrier instead of done, so the
//     peer's bounded wait for done runs out and neither CTA stores a partial accumulator;
//   - TMEM is allocated and freed by warp 2 of both CTAs together (cta_group::2), and a
//     cluster barrier orders the barrier initialisation and allocation before any load or MMA,
//     and every TMEM read of both CTAs before the free.
// Every CTA of the pair reaches both cluster barriers on every path (no early return).
template <int BN, int STAGES>
struct PairShape {
    static constexpr int WB = BN / 2;                       // W rows per CTA
    static constexpr int B_BYTES = WB * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int TMEM_COLS = BN < 32 ? 32 : BN;
    static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 + 256;
    static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "pair MMA: N a multiple of 16 per CTA half, at most 256");
};

template <int BN, int STAGES>
__global__ void __launch_bounds__(128, 1)
k_gemm_tc_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW, int M, int N, int K,
               Epi epi, EpiArgs ea, DevHeader* hdr) {
    using S = PairShape<BN, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * S::STAGE_BYTES);   // used in the leader
    uint64_t* empty = full + STAGES;
    uint64_t* done = empty + STAGES;
    uint64_t* drain = done + 1;               // leader: the MMAs issued before a timeout completed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    __shared__ int abort_flag, fin;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const int m0 = blockIdx.y * 2 * BM + (int)rank * BM;
    const int n0 = (blockIdx.x >> 1) * BN;
    const int nkb = (K + BK - 1) / BK;
    pdl_trigger();

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        mbar_init(drain, 1);
        abort_flag = 0;
        fin = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(S::TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    cluster_arrive_release();
    cluster_wait_acquire();                  // both CTAs' barriers initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // the MMA writes the peer's rows at the leader's TMEM address: both allocations must agree
    if (rank == 0 && threadIdx.x == 0 && dsmem_ld_u32(cluster_addr(tmem_slot, 1)) != tmem) abort_flag = 1;
    __syncthreads();

    const uint64_t lim = ea.wait_ns;
    int armed = 0;
    if (warp == 0 && lane == 0) {
        // producer of this CTA's halves; weight tiles before the programmatic-launch wait
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmA) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmW) : "memory");
        const uint32_t full0 = cluster_addr(full, 0);
        const int wrow = n0 + (int)rank * S::WB;
        const int pre = (ea.no_loads || abort_flag) ? 0 : (nkb < STAGES ? nkb : STAGES);
        for (int kb = 0; kb < pre; ++kb) {
            uint8_t* a = smem + kb * S::STAGE_BYTES;
            if (rank == 0) mbar_expect_tx(&full[kb], 2 * S::STAGE_BYTES);
            tma_load_2d_pair(a + A_BYTES, &tmW, full0 + 8u * kb, kb * BK, wrow);
        }
        pdl_wait();
        for (int kb = 0; kb < pre; ++kb) tma_load_2d_pair(smem + kb * S::STAGE_BYTES, &tmA, full0 + 8u * kb, kb * BK, m0);
        armed = pre;
        for (int kb = pre; kb < nkb && pre > 0; ++kb) {
            const int s = kb % STAGES;
            const uint32_t ph = (kb / STAGES) & 1;
            if (!mbar_wait(&empty[s], ph ^ 1, &abort_flag, lim)) { abort_flag = 1; break; }
            uint8_t* a = smem + s * S::STAGE_BYTES;
            if (rank == 0) mbar_expect_tx(&full[s], 2 * S::STAGE_BYTES);
            tma_load_2d_pair(a, &tmA, full0 + 8u * s, kb * BK, m0);
            tma_load_2d_pair(a + A_BYTES, &tmW, full0 + 8u * s, kb * BK, wrow);
            armed = kb + 1;
        }
    } else if (warp == 1 && lane == 0 && rank == 0) {
        // MMA issuer of the pair (leader only)
        constexpr uint32_t idesc = idesc_bf16(2 * BM, BN);
        for (int kb = 0; kb < nkb && !abort_flag; ++kb) {
            const int s = kb % STAGES;
            const uint32_t ph = (kb / STAGES) & 1;
            if (!mbar_wait(&full[s], ph, &abort_flag, lim)) { abort_flag = 1; break; }
            tc_fence_after();
            uint8_t* a = smem + s * S::STAGE_BYTES;
            const uint64_t da = sdesc_sw128(a), dw = sdesc_sw128(a + A_BYTES);
#pragma unroll
            for (int k = 0; k < BK / 16; ++k) umma_pair(tmem, da + 2 * k, dw + 2 * k, idesc, (kb | k) != 0);
            umma_commit_pair(&empty[s]);
        }
        // exactly one commit tracks every MMA issued (none in flight when TMEM is read or freed)
        if (abort_flag) {
            umma_commit_pair(drain, 1);
            fin = 2;
        } else if (nkb > 0) {
            umma_commit_pair(done, 3);
            fin = 1;
        }
    }
    __syncwarp();
    pdl_wait();

    RowNorm rn;
    const int m = m0 + warp * 32 + lane;
    if (ea.ss_in && m < M) rn.rinv = deferred_rinv(ea, m);
    // the leader stops waiting as soon as one of its roles gives up
    bool ok = nkb == 0 ? true : mbar_wait(done, 0, rank == 0 ? &abort_flag : nullptr, lim);
    ok = __syncthreads_and(ok) && abort_flag == 0;
    tc_fence_after();
    if (ok)
        epilogue_row<BN>(epi, ea, tmem + ((uint32_t)(warp * 32) << 16), m, M, n0, N, blockIdx.x >> 1, rn,
                         smem + warp * STG_BYTES);     // the consumed ring stages the epilogue
    if (!ok && threadIdx.x == 0) {
        raise_flag(hdr, ERR_TIMEOUT);
        if (rank == 0) {
            // the leader waits (bounded) for the MMAs it issued and for the stages it armed (a
            // peer's loads complete on them too)
            if (fin == 1) mbar_wait(done, 0, nullptr, lim);
            if (fin == 2) mbar_wait(drain, 0, nullptr, lim);
            for (int kb = armed > STAGES ? armed - STAGES : 0; kb < armed; ++kb)
                mbar_wait(&full[kb % STAGES], (kb / STAGES) & 1, nullptr, lim);
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_arrive_release();
    cluster_wait_acquire();                  // both CTAs have read their accumulators
    if (warp == 2) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(S::TMEM_COLS));
    }
}

// Persistent row-tile GEMM for grids of many waves (the encoder's projections, the LM head at
// large batch): one CTA per SM walks the 128 x BN output tiles (tile = blockIdx.x, then every
// gridDim.x-th; tiles ordered column-fastest, so that the CTAs in flight share the activation
// row tile in L2), with two TMEM accumulators so that the epilogue of one tile overlaps the
// MMAs of the next.  6 warps:
//   warp 0, lane 0   TMA producer over all k-blocks of all the CTA's tiles (one ring);
//   warp 1           allocates the 2 * BN TMEM columns; lane 0 issues the MMAs of tile i into
//                    accumulator i % 2 once the epilogue has drained it (acc_empty), then
//                    commits acc_full;
//   warps 2-9        epilogue: warp w reads TMEM lanes 32 * (w % 4) .. +31, i.e. output rows
//                    of that quadrant, and columns of half (w - 2) / 4 of the tile (the fused
//                    head's per-row reduction: warps 2-5 over all columns), with the fused
//                    epilogues of k_gemm_tc, then arrives on acc_empty.
// Every wait is bounded; after a timeout every role stops, the MMA issuer still commits what it
// issued, the CTA waits (bounded) for its loads in flight, latches ERR_TIMEOUT and stores
// nothing more.
constexpr int PERS_EPI_WARPS = 8;

template <int BN, int STAGES>
__global__ void __launch_bounds__((2 + PERS_EPI_WARPS) * 32, 1)
k_gemm_tc_pers(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW, int M, int N, int K,
               Epi epi, EpiArgs ea, DevHeader* hdr) {
    using S = TcShape<BN, STAGES, 1>;
    constexpr int ACC_COLS = 2 * BN;                 // two accumulators
    static_assert(ACC_COLS <= 512, "two accumulators must fit in TMEM");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * S::STAGE_BYTES);
    uint64_t* empty = full + STAGES;
    uint64_t* acc_full = empty + STAGES;             // [2]
    uint64_t* acc_empty = acc_full + 2;              // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
    // the epilogue warps' staging areas (the ring keeps loading the next tiles meanwhile)
    uint8_t* stg_all = smem + STAGES * S::STAGE_BYTES + 256;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mt = (M + BM - 1) / BM, nt = (N + BN - 1) / BN;
    const int tiles = mt * nt;
    const int nkb = (K + BK - 1) / BK;
    const uint64_t lim = ea.wait_ns;
    pdl_trigger();

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], PERS_EPI_WARPS);   // one arrival per epilogue warp
        }
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(ACC_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    int armed = 0;                                   // producer: k-blocks whose loads were issued

    if (warp == 0) {
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(&tmA) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(&tmW) : "memory");
            pdl_wait();
            int it = 0;
            for (int tile = blockIdx.x; tile < tiles && !ea.no_loads; tile += gridDim.x) {
                const int m0 = (tile / nt) * BM, n0 = (tile % nt) * BN;
                bool ok = true;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % STAGES;
                    if (it >= STAGES && !mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, &abort_flag, lim)) {
                        abort_flag = 1;
                        ok = false;
                        break;
                    }
                    uint8_t* a = smem + s * S::STAGE_BYTES;
                    mbar_expect_tx(&full[s], S::STAGE_BYTES);
                    tma_load_2d(a, &tmA, &full[s], kb * BK, m0);
                    tma_load_2d(a + A_BYTES, &tmW, &full[s], kb * BK, n0);
                    armed = it + 1;
                }
                if (!ok) break;
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(BM, BN);
            int it = 0, count = 0;
            for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++count) {
                const int a = count & 1, use = count >> 1;
                // accumulator a is free once the epilogue has drained its previous tile
                if (use > 0 && !mbar_wait(&acc_empty[a], (use - 1) & 1, &abort_flag, lim)) { abort_flag = 1; break; }
                tc_fence_after();
                bool ok = true;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % STAGES;
                    if (!mbar_wait(&full[s], (it / STAGES) & 1, &abort_flag, lim)) { abort_flag = 1; ok = false; break; }
                    tc_fence_after();
                    uint8_t* st = smem + s * S::STAGE_BYTES;
                    const uint64_t da = sdesc_sw128(st), dw = sdesc_sw128(st + A_BYTES);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        umma(tmem + a * BN, da + 2 * k, dw + 2 * k, idesc, (kb | k) != 0);
                    umma_commit(&empty[s]);
                }
                umma_commit(&acc_full[a]);           // also after a timeout: tracks what was issued
                if (!ok) break;
            }
        }
    } else {
        // epilogue warps: TMEM lane quadrant q = warp % 4 holds output rows 32q .. 32q+31
        pdl_wait();
        const int q = warp & 3, chalf = (warp - 2) / 4;
        int count = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++count) {
            const int a = count & 1, use = count >> 1;
            const int tm = tile / nt, tn = tile % nt;
            const int m0 = tm * BM, n0 = tn * BN;
            const int m = m0 + q * 32 + lane;
            RowNorm rn;
            if (ea.ss_in && m < M) rn.rinv = deferred_rinv(ea, m);
            bool ok = mbar_wait(&acc_full[a], use & 1, &abort_flag, lim);
            ok = __all_sync(0xffffffffu, ok) && abort_flag == 0;
            // the fused head's halves meet at a named barrier below: all eight epilogue warps
            // take the same decision (every one of them reaches this barrier: its wait is bounded)
            if (epi == Epi::LsePart) ok = bar_and(1, PERS_EPI_WARPS * 32, ok);
            if (!ok) { abort_flag = 1; break; }
            tc_fence_after();
            const uint32_t lane_base = tmem + a * BN + ((uint32_t)(q * 32) << 16);
            if (epi != Epi::LsePart) {
                epilogue_row<BN>(epi, ea, lane_base, m, M, n0, N, tn, rn, stg_all + (warp - 2) * STG_BYTES,
                                 chalf * (BN / 2), (chalf + 1) * (BN / 2));
            } else {
                // two halves of the columns, merged in column order through shared memory (two
                // buffers by tile parity: a buffer is rewritten only after the next barrier)
                const float2 part = lse_partial<BN>(ea, lane_base, m, M, n0, N, chalf * (BN / 2), (chalf + 1) * (BN / 2));
                float2* xbuf = reinterpret_cast<float2*>(stg_all) + (count & 1) * BM;
                if (chalf == 1) xbuf[q * 32 + lane] = part;
                asm volatile("bar.sync 1, %0;" ::"r"(PERS_EPI_WARPS * 32) : "memory");
                if (chalf == 0 && m < M) ea.lse_part[(long long)m * ea.lse_ld + tn] = lse_merge(part, xbuf[q * 32 + lane]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[a]);
        }
    }
    __syncwarp();
    // a role that gave up raised abort_flag before this barrier
    const bool ok = __syncthreads_and(1) && abort_flag == 0;
    if (!ok && threadIdx.x == 0) {
        raise_flag(hdr, ERR_TIMEOUT);
        for (int it = armed > STAGES ? armed - STAGES : 0; it < armed; ++it)
            mbar_wait(&full[it % STAGES], (it / STAGES) & 1, nullptr, lim);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ACC_COLS));
    }
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void* p = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D bf16 tensor [rows, cols] with leading dimension ld (elements), box of BK x box_rows.
bool make_map(CUtensorMap* map, const void* ptr, int rows, int cols, int ld, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Host cache of encoded tensor maps: weights and workspaces keep their addresses and shapes
// across steps, so each (address, shape, box) is encoded once.
struct MapKey {
    const void* p;
    int rows, cols, ld, box;
    bool operator==(const MapKey& o) const {
        return p == o.p && rows == o.rows && cols == o.cols && ld == o.ld && box == o.box;
    }
};
struct MapKeyHash {
    size_t operator()(const MapKey& k) const {
        size_t h = std::hash<const void*>()(k.p);
        for (int v : {k.rows, k.cols, k.ld, k.box}) h = h * 1000003u ^ std::hash<int>()(v);
        return h;
    }
};

bool cached_map(CUtensorMap* map, const void* ptr, int rows, int cols, int ld, int box_rows) {
    static std::mutex mu;
    static std::unordered_map<MapKey, CUtensorMap, MapKeyHash> cache;
    MapKey k{ptr, rows, cols, ld, box_rows};
    std::lock_guard<std::mutex> g(mu);
    auto it = cache.find(k);
    if (it != cache.end()) {
        *map = it->second;
        return true;
    }
    if (!make_map(map, ptr, rows, cols, ld, box_rows)) return false;
    if (cache.size() > 8192) cache.clear();
    cache.emplace(k, *map);
    return true;
}

}  // namespace

bool tma_map_bf16(CUtensorMap* map, const void* ptr, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
                  const uint32_t* box) {
    struct Key {
        const void* p;
        int rank;
        uint64_t d[5], s[4];
        uint32_t b[5];
        bool operator==(const Key& o) const { return std::memcmp(this, &o, sizeof(Key)) == 0; }
    };
    struct Hash {
        size_t operator()(const Key& k) const {
            const unsigned char* c = reinterpret_cast<const unsigned char*>(&k);
            size_t h = 1469598103934665603ull;
            for (size_t i = 0; i < sizeof(Key); ++i) h = (h ^ c[i]) * 1099511628211ull;
            return h;
        }
    };
    static std::mutex mu;
    static std::unordered_map<Key, CUtensorMap, Hash> cache;
    if (rank < 1 || rank > 5) return false;
    Key k;
    std::memset(&k, 0, sizeof(k));
    k.p = ptr;
    k.rank = rank;
    for (int i = 0; i < rank; ++i) { k.d[i] = dims[i]; k.b[i] = box[i]; }
    for (int i = 0; i + 1 < rank; ++i) k.s[i] = strides_bytes[i];
    std::lock_guard<std::mutex> g(mu);
    auto it = cache.find(k);
    if (it != cache.end()) {
        *map = it->second;
        return true;
    }
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gd[5], gs[4];
    cuuint32_t bx[5], es[5];
    for (int i = 0; i < rank; ++i) { gd[i] = dims[i]; bx[i] = box[i]; es[i] = 1; }
    for (int i = 0; i + 1 < rank; ++i) gs[i] = strides_bytes[i];
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(ptr), gd, gs, bx, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    if (cache.size() > 8192) cache.clear();
    cache.emplace(k, *map);
    return true;
}

namespace {

template <int BN, int STAGES, int SPLIT, int KA = 1, int EW = 4>
cudaError_t run_tc(Launch L, Epi epi, const bf16* A, int lda, const bf16* W, int M, int N, int K, const EpiArgs& ea,
                   DevHeader* hdr) {
    using S = TcShape<BN, STAGES, SPLIT, KA>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(k_gemm_tc<BN, STAGES, SPLIT, KA, EW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             S::SMEM);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    CUtensorMap ta, tw;
    if (!cached_map(&ta, A, M, K, lda, BM) || !cached_map(&tw, W, N, K, K, BN)) return cudaErrorInvalidValue;
    dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM, SPLIT);
    if constexpr (SPLIT == 1) {
        return launch_k(L, k_gemm_tc<BN, STAGES, 1, KA, EW>, grid, EW * 32, S::SMEM, ta, tw, M, N, K, epi, ea, hdr);
    } else {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = grid;
        cfg.blockDim = dim3(128);
        cfg.dynamicSmemBytes = S::SMEM;
        cfg.stream = L.stream;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 1;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = SPLIT;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = L.pdl ? 1 : 0;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        *L.count += 1;
        return cudaLaunchKernelEx(&cfg, k_gemm_tc<BN, STAGES, SPLIT, KA, 4>, ta, tw, M, N, K, epi, ea, hdr);
    }
}

// The CTA-pair kernel: clusters of two CTAs along x, one 256-row band of tiles per grid row.
template <int BN, int STAGES>
cudaError_t run_tc_pair(Launch L, Epi epi, const bf16* A, int lda, const bf16* W, int M, int N, int K,
                        const EpiArgs& ea, DevHeader* hdr) {
    using S = PairShape<BN, STAGES>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(k_gemm_tc_pair<BN, STAGES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             S::SMEM);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    CUtensorMap ta, tw;
    if (!cached_map(&ta, A, M, K, lda, BM) || !cached_map(&tw, W, N, K, K, S::WB)) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * ((N + BN - 1) / BN), (M + 2 * BM - 1) / (2 * BM), 1);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = S::SMEM;
    cfg.stream = L.stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = L.pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    *L.count += 1;
    return cudaLaunchKernelEx(&cfg, k_gemm_tc_pair<BN, STAGES>, ta, tw, M, N, K, epi, ea, hdr);
}

// The persistent kernel for grids of more than one wave: one CTA per SM.
template <int BN, int STAGES>
cudaError_t run_tc_pers(Launch L, Epi epi, const bf16* A, int lda, const bf16* W, int M, int N, int K,
                        const EpiArgs& ea, DevHeader* hdr) {
    using S = TcShape<BN, STAGES, 1>;
    constexpr int SMEM = STAGES * S::STAGE_BYTES + 1024 + 256 + PERS_EPI_WARPS * STG_BYTES;   // + epilogue staging
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(k_gemm_tc_pers<BN, STAGES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             SMEM);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    CUtensorMap ta, tw;
    if (!cached_map(&ta, A, M, K, lda, BM) || !cached_map(&tw, W, N, K, K, BN)) return cudaErrorInvalidValue;
    const long long tiles = (long long)((M + BM - 1) / BM) * ((N + BN - 1) / BN);
    const unsigned grid = (unsigned)(tiles < sm_count() ? tiles : sm_count());
    return launch_k(L, k_gemm_tc_pers<BN, STAGES>, grid, (2 + PERS_EPI_WARPS) * 32, SMEM, ta, tw, M, N, K, epi, ea, hdr);
}

// Tile variants: (BN, stages, CTAs per SM, k-split over a cluster, 64-wide k-atoms per stage);
// the one-per-SM 128- and 256-wide unsplit tiles run their epilogue on eight warps.
// Two atoms per stage where it measured faster at decode sizes (B200, 512 x 1024 x 1024:
// 128x64 split 2 7.06 -> 6.28 us; 512 x 3072 x 1024: 128x128 9.85 -> 8.51 us; 64 x 2048 x 2048:
// 128x64 split 4 7.35 -> 6.61 us); the 256-wide tile is bound by its MMAs and keeps one.
struct TcVariant {
    int bn, stages, per_sm, split, ka;
};
constexpr TcVariant VARIANTS[] = {
    // Decode-size grids run one CTA per SM, so the rings fill ~200 KB of shared memory.
    {32, 5, 1, 1, 2},     // 200 KB
    {64, 4, 1, 1, 2},     // 192 KB
    {128, 3, 2, 1, 1},    //  96 KB (two CTAs per SM for grids of up to two waves)
    {128, 3, 1, 1, 2},    // 192 KB
    {256, 4, 1, 1, 1},    // 192 KB
    {128, 4, 1, 2, 1},    // 128 KB + 64 KB partials
    {128, 2, 1, 4, 2},    // 128 KB + 64 KB
    {64, 3, 1, 2, 2},     // 144 KB + 32 KB partials
    {64, 3, 1, 4, 2},     // 144 KB + 32 KB
};
constexpr int N_VARIANTS = sizeof(VARIANTS) / sizeof(VARIANTS[0]);

cudaError_t run_variant(int v, Launch L, Epi epi, const bf16* A, int lda, const bf16* W, int M, int N, int K,
                        const EpiArgs& ea, DevHeader* hdr) {
    switch (v) {
        case 0: return run_tc<32, 5, 1, 2>(L, epi, A, lda, W, M, N, K, ea, hdr);
        case 1: return run_tc<64, 4, 1, 2>(L, epi, A, lda, W, M, N, K, ea, hdr);
        case 2: return run_tc<128, 3, 1, 1>(L, epi, A, lda, W, M, N, K, ea, hdr);
        case 3: return run_tc<128, 3, 1, 2, 8>(L, epi, A, lda, W, M, N, K, ea, hdr);
        case 4: return run_tc<256, 4, 1, 1, 8>(L, epi, A, lda, W, M, N, K, ea, hdr);
        case 5: return run_tc<128, 4, 2, 1>(L, epi, A, lda, W, M, N, K, ea, hdr);
        case 6: return run_tc<128, 2, 4, 2>(L, epi, A, lda, W, M, N, K, ea, hdr);
        case 7: return run_tc<64, 3, 2, 2>(L, epi, A, lda, W, M, N, K, ea, hdr);
        case 8: return run_tc<64, 3, 4, 2>(L, epi, A, lda, W, M, N, K, ea, hdr);
    }
    return cudaErrorInvalidValue;
}

// At decode sizes one CTA per output tile leaves a latency-bound k-loop: the widest
// unsplit tile whose grid fits in one wave (and keeps at least half the SMs busy) with at most
// 16 k-blocks per CTA wins; otherwise the k-blocks are split over a cluster so that the grid
// fills one wave with as few k-blocks per CTA as possible.  Grids larger than a wave use the
// widest tile.
int pick_variant(int M, int N, int K) {
    long long mt = (M + BM - 1) / BM;
    int nkb = (K + BK - 1) / BK;
    for (int v = 4; v >= 0; --v) {
        const TcVariant& t = VARIANTS[v];
        long long tiles = mt * ((N + t.bn - 1) / t.bn);
        if (tiles <= 148LL * t.per_sm && tiles >= 74 && nkb <= 16) {
            // 32-wide tiles re-read the activation panel from L2 for every 32 output columns;
            // 64-wide tiles with K split in two give as many CTAs for half that traffic
            if (v == 0 && mt * ((N + 63) / 64) * 2 <= 148 && nkb >= 8) return 7;
            return v;
        }
    }
    long long tiles256 = mt * ((N + 255) / 256);
    if (tiles256 > 148) return 4;
    int best = -1;
    long long best_ctas = 0;
    for (int v = 5; v < N_VARIANTS; ++v) {
        const TcVariant& t = VARIANTS[v];
        long long ctas = mt * ((N + t.bn - 1) / t.bn) * t.split;
        if (ctas > 148 || t.split * t.ka > nkb) continue;
        if (ctas > best_ctas) { best = v; best_ctas = ctas; }
    }
    if (best >= 0 && best_ctas >= 64) return best;
    // fall back to the unsplit tile with the most CTAs within a wave
    for (int v = 0; v <= 4; ++v) {
        const TcVariant& t = VARIANTS[v];
        if (mt * ((N + t.bn - 1) / t.bn) <= 148LL * t.per_sm) return v;
    }
    return 4;
}

}  // namespace

int gemm_tc_variants() { return N_VARIANTS; }

int gemm_tc_pick(int M, int N, int K) { return pick_variant(M, N, K); }

bool gemm_tc_supported(const void* A, int lda, const void* W, int K) {
    // TMA: 16-byte aligned base addresses and row pitches
    return (reinterpret_cast<uintptr_t>(A) % 16 == 0) && (reinterpret_cast<uintptr_t>(W) % 16 == 0) &&
           (lda % 8 == 0) && (K % 8 == 0) && encode_fn() != nullptr;
}

// Whether a 128 x 256 grid of this shape takes more than one wave (the persistent kernel's case).
bool multi_wave_256(int M, int N) {
    return (long long)((M + BM - 1) / BM) * ((N + 255) / 256) > sm_count();
}

cudaError_t launch_gemm_tc_lse(Launch L, const bf16* A, int lda, const bf16* W, int M, int N, int K, EpiArgs ea,
                               DevHeader* hdr, int* n_tiles) {
    int v = pick_variant(M, N, K);
    if (VARIANTS[v].split > 1) v = 4;                 // the fused head needs whole rows per CTA
    ea.lse_ld = (N + VARIANTS[v].bn - 1) / VARIANTS[v].bn;
    *n_tiles = ea.lse_ld;
    if (v == 4 && multi_wave_256(M, N)) return run_tc_pers<256, 4>(L, Epi::LsePart, A, lda, W, M, N, K, ea, hdr);
    return run_variant(v, L, Epi::LsePart, A, lda, W, M, N, K, ea, hdr);
}

cudaError_t launch_gemm_tc(Launch L, Epi epi, const bf16* A, int lda, const bf16* W, int M, int N, int K,
                           const EpiArgs& ea, DevHeader* hdr, int variant) {
    if (variant == PERSISTENT_VARIANT) return run_tc_pers<256, 4>(L, epi, A, lda, W, M, N, K, ea, hdr);
    switch (variant) {      // CTA-pair tiles 256 x 64 / 128 / 256 (stages: ~200 KB of ring per CTA)
        case PAIR_VARIANT + 0: return run_tc_pair<64, 10>(L, epi, A, lda, W, M, N, K, ea, hdr);
        case PAIR_VARIANT + 1: return run_tc_pair<128, 8>(L, epi, A, lda, W, M, N, K, ea, hdr);
        case PAIR_VARIANT + 2: return run_tc_pair<256, 6>(L, epi, A, lda, W, M, N, K, ea, hdr);
        default: break;
    }
    int v = (variant >= 0 && variant < N_VARIANTS) ? variant : pick_variant(M, N, K);
    // a merge's deferred-norm group spans 32 GEMM columns and must stay in one column band
    if (epi == Epi::Merge && ea.norm_y && VARIANTS[v].split > 1 && VARIANTS[v].bn / VARIANTS[v].split < 32) v = 7;
    // grids of several waves of the widest tile run persistently (epilogue overlapped)
    if (variant < 0 && v == 4 && L.persistent && multi_wave_256(M, N))
        return run_tc_pers<256, 4>(L, epi, A, lda, W, M, N, K, ea, hdr);
    return run_variant(v, L, epi, A, lda, W, M, N, K, ea, hdr);
}

}  // namespace rlt
