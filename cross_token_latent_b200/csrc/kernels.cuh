// Host-side launchers of the RLT kernels.  Every launcher enqueues exactly the kernels
// it names on `L.stream`, adds their number to *L.count and returns the launch status.
#pragma once

#include <utility>

#include "common.cuh"

namespace rlt {

struct Launch {
    cudaStream_t stream;
    uint64_t* count;
    // Programmatic dependent launch (see pdl_wait in common.cuh).  Off when two row groups of
    // a step run on two streams: a kernel launched early would hold its SM resources while it
    // waits, which the other group's kernels need.
    bool pdl = true;
    // Cap on the resident CTAs per SM of the attention kernels (0: none).  With two row groups
    // the attention of one group leaves room on every SM for the other group's projections.
    int attn_ctas_per_sm = 0;
    // Projections with at most this many rows of A run on the weight-streaming CUDA-core kernel
    // (gemv.cu) when its shape rules hold (0: never).
    int gemv_max_rows = 0;
    // Grids of several waves of 128 x 256 tiles run on the persistent row-tile kernel.
    bool persistent = true;
};

// Number of SMs of the current device (queried once per process).
inline int sm_count() {
    static int n = 0;
    if (n == 0) {
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
            n = v;
        else
            return 148;
    }
    return n;
}

// Launch `kernel` on L.stream (with programmatic stream serialization unless L.pdl is off)
// and count it.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(Launch L, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                            Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = L.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = L.pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    *L.count += 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ------------------------------------------------------------------ elementwise.cu
// dst[(r*row_mult + row_off) * dst_ld + col_off + c] = T(src[r*cols + c])
template <typename T>
cudaError_t launch_pack_rows(Launch L, const float* src, T* dst, int rows, int cols, int dst_ld,
                             int row_mult, int row_off, int col_off);
// table[p*half + i] = (cos, sin)(p * base^(-2i/hd)), computed in double precision
cudaError_t launch_rope_table(Launch L, float2* table, int max_pos, int head_dim, float base);
// h[n, :] = embed[tok[n * tok_stride], :] in float32
template <typename T>
cudaError_t launch_embed(Launch L, const int32_t* tok, int N, const T* embed, int V, int d, float* h,
                         DevHeader* hdr, int tok_stride = 1);
// out[row_map(n), out_col_off + :] = T(RMSNorm(x[n, :]) * gain).  row_map(n) =
// (n / rows_per_seq) * out_rows_per_seq + n % rows_per_seq; out2 (optional) is a second
// contiguous T copy with leading dimension d.
// With row_pos (device, one entry per row; rows_per_seq must be 1) row n lands at
// n * out_rows_per_seq + row_pos[n] instead.
template <typename T>
cudaError_t launch_rmsnorm(Launch L, const float* x, int N, int d, const float* gain, float eps,
                           T* out, int out_ld, int rows_per_seq, int out_rows_per_seq, T* out2,
                           const int32_t* row_pos = nullptr);
// A[b, :] = [e[b, pos[b], :] | T(s[b, :])] (the step of sequence b consumes its token at
// 0-based position pos[b]); also checks the state header and the position's range
template <typename T>
cudaError_t launch_merge_prep(Launch L, const T* e, int T_alloc, const int32_t* pos, const float* s, T* A, int B,
                              int d, const StateHeader* sh, uint64_t version, DevHeader* hdr);
// s[b, :] = RMSNorm(x[b, :]) * gain (float32) and hs = T(s); pos[b] += 1; sets the state
// header's t (the batch's largest position) when sh is given
template <typename T>
cudaError_t launch_final_norm(Launch L, const float* x, int B, int d, const float* gain, float eps,
                              float* s, T* hs, StateHeader* sh, int t, int32_t* pos);
// Per row b: z = logits[b, :] / tau, lse = logsumexp(z), gather z[tok] - lse, optional full
// row, optional score accumulation when the step t = pos[b] (positions after the step's
// advance) is at least P[b].
cudaError_t launch_lse_gather(Launch L, const float* logits, int B, int V, float tau,
                              const int32_t* tok, int tok_stride, float* logp_tok, int lp_stride,
                              float* lse, float* logp_full, float* score, const int32_t* prompt_len,
                              const int32_t* pos, DevHeader* hdr);
// Per row b: LSE = log sum_j part.y exp(part.x - max) + max over the n_tiles column-tile
// partials of the fused head; the gathered log-prob z_tok[b] - LSE, the LSE itself and the
// score accumulation as in launch_lse_gather (bad token ids latch ERR_BAD_TOKEN).
cudaError_t launch_lse_combine(Launch L, const float2* part, int n_tiles, const float* z_tok, int B, int V,
                               const int32_t* tok, int tok_stride, float* logp_tok, int lp_stride, float* lse,
                               float* score, const int32_t* prompt_len, const int32_t* pos, DevHeader* hdr);
// Encoder q/k/v: qkv float32 [B*T, 3d] -> planes T [3][B][H][T][hd], RoPE on q and k; the v
// plane is skipped when write_v is false (the tensor-core path writes V transposed instead).
template <typename T>
cudaError_t launch_enc_qkv_layout(Launch L, const float* qkv, int B, int Tn, int H, int hd,
                                  const float2* rope, T* planes, bool write_v = true);
// Memory projection output float32 [B*T, 2d] -> M_g T [2][B][H][T_alloc][hd]; with row_pos
// (Tn = 1) sequence b's row lands at position row_pos[b]
template <typename T>
cudaError_t launch_mem_layout(Launch L, const float* kv, int B, int Tn, int T_alloc, int H, int hd,
                              T* Mg, const int32_t* row_pos = nullptr);
// Encoder key/value cache of one layer [2][B][H][T_max][hd]: rotated keys and values of the Tn
// tokens of qkv float32 [B*Tn, 3d] at positions pos0 .. pos0+Tn-1, in the storage type; with
// q_out (Tn = 1) also the rotated, storage-rounded query as float32 [B, d].
// With row_pos (device, Tn = 1) sequence b's token is at position row_pos[b] instead.
template <typename T>
cudaError_t launch_enc_cache_write(Launch L, const float* qkv, int B, int Tn, int H, int hd, const float2* rope,
                                   int pos0, const int32_t* row_pos, T* cache_l, int T_max, float* q_out);
// H_0: s[b, :] = s_star, pos[b] = 0, header (t=0, version, B); with row >= 0 only that row's s
// and position (the header is left alone)
cudaError_t launch_state_init(Launch L, const float* s_star, int B, int d, float* s, StateHeader* sh,
                              uint64_t version, int32_t* pos, int row = -1);

// ------------------------------------------------------------------ gemm_simt.cu
// C[M, N] = A[M, K] (leading dim lda) x W[N, K]^T, float32 accumulation, then an epilogue.
enum class Epi { StoreF32, ResidAdd, SwiGLU, Merge, LsePart };
struct EpiArgs {
    float* out_f32 = nullptr;   // StoreF32 target / ResidAdd accumulator / Merge output x
    void* out_t = nullptr;      // SwiGLU output (storage type)
    int ld_out = 0;
    float scale = 1.0f;         // StoreF32 multiplier
    const void* merge_e = nullptr;  // Merge: e_t rows (storage type), leading dim ld_e
    int ld_e = 0;
    const float* bias = nullptr;    // Merge: gate bias b_g
    DevHeader* hdr = nullptr;       // error flags (tensor-core path: bounded-wait timeouts)
    // Tensor-core kernels: limit of every mbarrier wait (%globaltimer nanoseconds).  no_loads is
    // the bounded-wait self-test: the kernel issues no TMA load and no MMA, so its first wait
    // runs out after wait_ns and the launch latches ERR_TIMEOUT without writing any output.
    unsigned long long wait_ns = 2000000000ull;
    int no_loads = 0;
    // Deferred RMSNorm (tensor-core paths only; the output width is a multiple of 16).
    // Producer side (ResidAdd, Merge): with norm_y set, the epilogue also writes
    // norm_y[m][c] = bf16(x_new[m][c] * norm_g[c]) (leading dim ld_out) and, for every group of
    // 16 consecutive output columns, ss_out[m * ss_ld + c / 16] = sum of x_new^2 over the group
    // (one writer per group, fixed summation order).
    bf16* norm_y = nullptr;
    const float* norm_g = nullptr;
    float* ss_out = nullptr;
    // Consumer side: with ss_in set, accumulator row m is multiplied by
    // 1 / sqrt(sum_{g < ss_n} ss_in[m * ss_ld + g] / norm_n + eps) before the epilogue, i.e. the
    // GEMM of bf16(x * g) becomes the GEMM of RMSNorm(x) * g.
    const float* ss_in = nullptr;
    int ss_ld = 0, ss_n = 0;
    float norm_n = 1.f, eps = 0.f;
    // LM head with a fused log-sum-exp (LsePart, row-tile tensor-core kernel without a K
    // split): with z = acc * scale, the CTA of column tile j writes, for each of its rows m,
    // lse_part[m * lse_ld + j] = (max of z over the tile's columns, sum of exp(z - max)); the
    // tile holding column lse_tok[m * tok_stride] (an id outside [0, N) counts as 0) writes
    // z_tok[m].  No logits are stored.
    const int32_t* lse_tok = nullptr;
    int tok_stride = 1;
    float2* lse_part = nullptr;
    int lse_ld = 0;
    float* z_tok = nullptr;
};
// 1 / rms of row m from its 16-column group partials (summed in group order).
__device__ __forceinline__ float deferred_rinv(const EpiArgs& ea, long long m) {
    const float* p = ea.ss_in + m * ea.ss_ld;
    float s = 0.f;
    for (int g = 0; g < ea.ss_n; g += 4) {
        float4 q = *reinterpret_cast<const float4*>(p + g);
        s += q.x; s += q.y; s += q.z; s += q.w;
    }
    return 1.0f / sqrtf(s / ea.norm_n + ea.eps);
}
// Dispatch: bf16 operands go to the tcgen05 kernel (gemm_tc.cu) when TMA can address them,
// otherwise (and for float32 models) to the CUDA-core kernel.
template <typename T>
cudaError_t launch_gemm(Launch L, Epi epi, const T* A, int lda, const T* W, int M, int N, int K,
                        const EpiArgs& ea);
template <typename T>
cudaError_t launch_gemm_simt(Launch L, Epi epi, const T* A, int lda, const T* W, int M, int N, int K,
                             const EpiArgs& ea);

// ------------------------------------------------------------------ gemm_tc.cu
bool gemm_tc_supported(const void* A, int lda, const void* W, int K);
int gemm_tc_variants();
// launch_gemm_tc's variant id of the persistent 128 x 256 kernel (two TMEM accumulators)
constexpr int PERSISTENT_VARIANT = 100;
// launch_gemm_tc's variant ids of the CTA-pair kernel: PAIR_VARIANT + p, tiles 256 x (64 << p)
constexpr int PAIR_VARIANT = 200;
constexpr int N_PAIR_VARIANTS = 3;
// the row-tile variant the library picks for an M x N x K product (host logic only)
int gemm_tc_pick(int M, int N, int K);
// variant < 0: pick the tile shape from (M, N); otherwise force tile variant `variant`.
cudaError_t launch_gemm_tc(Launch L, Epi epi, const bf16* A, int lda, const bf16* W, int M, int N, int K,
                           const EpiArgs& ea, DevHeader* hdr, int variant = -1);

// The LM head with the fused log-sum-exp epilogue (Epi::LsePart, M > 64): picks an unsplit
// row-tile variant, sets ea.lse_ld to its number of column tiles and launches it; *n_tiles
// receives that number for launch_lse_combine.
cudaError_t launch_gemm_tc_lse(Launch L, const bf16* A, int lda, const bf16* W, int M, int N, int K, EpiArgs ea,
                               DevHeader* hdr, int* n_tiles);

// ------------------------------------------------------------------ gemm_swap.cu
// Few-row products (1 <= M <= 64) with the weights on the MMA's M side; split = K split over a
// cluster of 1, 2, 4 or 8 CTAs (0: choose).
bool gemm_swap_supported(int M);
bool gemm_swap_preferred(int M, int N, int K);
// the K split (1, 2 or 4) the few-row kernel picks when asked to choose (host logic only)
int gemm_swap_auto_split(int M, int N, int K);
cudaError_t launch_gemm_swap(Launch L, Epi epi, const bf16* A, int lda, const bf16* W, int M, int N, int K,
                             const EpiArgs& ea, DevHeader* hdr, int split = 0);

// ------------------------------------------------------------------ gemv.cu
// Weight-streaming projection for 1..4 rows on CUDA cores, bulk-copied weight rows (requested
// before the programmatic-launch wait), the same fused epilogues.  Shape rules: N a multiple of
// 32, K a multiple of 8 and at most 6144, 16-byte aligned operands.
bool gemv_shape_supported(int M, int N, int K, int lda);
// the shapes where it measured faster than the few-row tensor-core kernel
bool gemv_preferred(int M, int N, int K);
bool gemv_supported(int M, int N, int K, int lda, const void* A, const void* W);
cudaError_t launch_gemv(Launch L, Epi epi, const bf16* A, int lda, const bf16* W, int M, int N, int K,
                        const EpiArgs& ea, DevHeader* hdr);

// ------------------------------------------------------------------ attention.cu
// Decoder sliding-window self-attention for one layer: sequence b is at step t = pos[b] + 1
// (clamped to 1 .. max_t): RoPE at position t-1 (rows of the rotary table `rope`) on q/k from
// qkv [B, 3d]; attends over the min(t-1, W-1) cached entries plus the current token; then
// stores k_t, v_t into ring slot (t-1) mod (W-1).  With n_splits > 1 the cached entries of
// each (b, h) are cut into n_splits ranges, one CTA each, whose partials (in `part`, as for
// the cross-attention) a combine kernel merges.
template <typename T>
cudaError_t launch_swa_decode(Launch L, const float* qkv, const float2* rope, T* ring, T* o,
                              int B, int H, int hd, int W, const int32_t* pos, int max_t,
                              int n_splits = 1, float* part = nullptr);
// Decoder cross-attention over M_{<=t} (positions 0..t-1) of one memory group: keys of
// (b, h) at Mg + (b*H + h)*T_alloc*hd, values `plane` elements further.  With pos (device,
// [B]) sequence b reads only positions 0..pos[b] (at most t).  Splits the keys of each (b, h)
// into n_splits chunks of ceil(t / n_splits) when n_splits > 1 (partials in `part`).
template <typename T>
cudaError_t launch_xattn_decode(Launch L, const float* qc, const T* Mg, long long plane, int T_alloc, int t,
                                T* o, int B, int H, int hd, int n_splits, float* part,
                                const int32_t* pos = nullptr);
// Encoder causal self-attention: planes T [3][B][H][T][hd] -> o T [B*T, d]
template <typename T>
cudaError_t launch_enc_attention(Launch L, const T* planes, T* o, int B, int Tn, int H, int hd);

// ------------------------------------------------------------------ sample.cu
// Largest vocabulary the sampler handles (its row lives in shared memory).
int sample_max_vocab();
// One token per row of logp [B, V] (log-probabilities at the sampling temperature) with the
// uniform u[b]: top-k / top-p truncation (ties at a boundary kept), inverse CDF over the kept
// tokens in id order.  tok[b * tok_stride] = the draw, blp[b] (optional) = its log-probability
// under the truncated, renormalised distribution.
cudaError_t launch_sample(Launch L, const float* logp, int B, int V, const float* u, int top_k, float top_p,
                          int32_t* tok, int tok_stride, float* blp);

// ------------------------------------------------------------------ small_step.cu
// The whole decoder step of a small model in one launch, one CTA per sequence.
constexpr int SS_MAX_LAYERS = 8;
struct DecWeights {             // device pointers into the weight arena (matrices in storage type)
    const void* merge;          // [2d, 2d], rows 2j / 2j+1 = gate_j / feedback_j
    const float* merge_b;
    const float* dec_norm;
    const void* unembed;        // [V, d]
    const float* attn_norm[SS_MAX_LAYERS];
    const float* xattn_norm[SS_MAX_LAYERS];
    const float* ffn_norm[SS_MAX_LAYERS];
    const void* wqkv[SS_MAX_LAYERS];
    const void* wo[SS_MAX_LAYERS];
    const void* wqc[SS_MAX_LAYERS];
    const void* woc[SS_MAX_LAYERS];
    const void* wgu[SS_MAX_LAYERS];     // [2F, d], rows 2j / 2j+1 = gate_j / up_j
    const void* wdown[SS_MAX_LAYERS];
};
struct SmallStepArgs {
    int B, d, H, F, V, W, G, L;
    float eps, tau;
    const void* e;              // [B, T_alloc, d]
    int T_alloc;
    const void* M;              // [G][2][B][H][T_alloc][hd]
    long long plane;            // keys -> values of one memory group
    size_t group_elems;
    float* s;                   // state s [B, d]
    void* ring;                 // state ring [L][B][2][H][W-1][hd]
    size_t ring_layer;          // elements per layer of the ring
    int32_t* pos;               // state positions [B]
    StateHeader* sh;
    int t_host;                 // the largest step of the batch (the header's t)
    uint64_t version;
    DevHeader* hdr;
    const float2* rope;
    DecWeights w;
    bool head;
    const int32_t* tok;
    int tok_stride;
    float* logp_tok;
    int lp_stride;
    float* lse;
    float* logp_full;
    float* score;
    const int32_t* prompt_len;
};
bool small_step_supported(int d, int F, int V, int hd, int L);
template <typename T>
cudaError_t launch_small_step(Launch L, const SmallStepArgs& a, int hd);

// ------------------------------------------------------------------ attention_tc.cu
// Tensor-core encoder attention (bf16, head_dim 64 or 128): q, k planes [B][H][T][hd] and the
// transposed values vt [B][H][hd][enc_vt_pitch(T)] -> o [B*T, d].
bool enc_attention_tc_supported(int hd);
int enc_vt_pitch(int Tn);
cudaError_t launch_enc_vt(Launch L, const float* qkv, bf16* vt, int B, int Tn, int H, int hd);
cudaError_t launch_enc_attention_tc(Launch L, const bf16* q, const bf16* k, const bf16* vt, bf16* o, int B, int Tn,
                                    int H, int hd, DevHeader* hdr);

}  // namespace rlt
