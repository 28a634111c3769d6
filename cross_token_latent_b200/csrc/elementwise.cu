// Bandwidth-bound elementwise kernels of the RLT path: weight packing, rotary table,
// embedding gather, RMSNorm, merge input assembly, final norm, fused log-softmax gather,
// and the layout kernels of the encoder.
#include "kernels.cuh"

namespace rlt {

namespace {

inline unsigned cdiv(long long a, long long b) { return (unsigned)((a + b - 1) / b); }

template <typename T>
__global__ void k_pack_rows(const float* __restrict__ src, T* __restrict__ dst, int rows, int cols,
                            int dst_ld, int row_mult, int row_off, int col_off) {
    pdl_wait();
    pdl_trigger();
    long long n = (long long)rows * cols;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x) {
        int r = (int)(i / cols), c = (int)(i % cols);
        dst[((long long)r * row_mult + row_off) * dst_ld + col_off + c] = from_f<T>(src[i]);
    }
}

__global__ void k_rope_table(float2* table, int max_pos, int half, int hd, double base) {
    pdl_wait();
    pdl_trigger();
    long long n = (long long)max_pos * half;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x) {
        int p = (int)(i / half), f = (int)(i % half);
        double inv = pow(base, -2.0 * f / hd);
        double s, c;
        sincos((double)p * inv, &s, &c);
        table[i] = make_float2((float)c, (float)s);
    }
}

template <typename T>
__global__ void k_embed(const int32_t* __restrict__ tok, int tok_stride, int N, const T* __restrict__ embed, int V,
                        int d, float* __restrict__ h, DevHeader* hdr) {
    pdl_wait();
    pdl_trigger();
    int n = blockIdx.x;
    if (n >= N) return;
    int id = tok[(long long)n * tok_stride];
    if (id < 0 || id >= V) {
        if (threadIdx.x == 0) raise_flag(hdr, ERR_BAD_TOKEN);
        id = 0;
    }
    const T* row = embed + (long long)id * d;
    float* out = h + (long long)n * d;
    for (int c = threadIdx.x; c < d; c += blockDim.x) out[c] = to_f(row[c]);
}

// One warp per row.  d is a multiple of 8, so float4 loads cover the row exactly.
template <typename T>
__global__ void k_rmsnorm(const float* __restrict__ x, int N, int d, const float* __restrict__ gain,
                          float eps, T* __restrict__ out, int out_ld, int rows_per_seq,
                          int out_rows_per_seq, T* __restrict__ out2, const int32_t* __restrict__ row_pos) {
    pdl_wait();
    pdl_trigger();
    int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    int lane = threadIdx.x & 31;
    if (warp >= N) return;
    const float4* xr = reinterpret_cast<const float4*>(x + (long long)warp * d);
    float ss = 0.f;
    for (int c = lane; c < d / 4; c += 32) {
        float4 v = xr[c];
        ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
    ss = warp_sum(ss);
    float r = 1.0f / sqrtf(ss / d + eps);
    long long orow = row_pos ? (long long)warp * out_rows_per_seq + min(max(row_pos[warp], 0), out_rows_per_seq - 1)
                             : (long long)(warp / rows_per_seq) * out_rows_per_seq + warp % rows_per_seq;
    T* o = out + orow * out_ld;
    T* o2 = out2 ? out2 + (long long)warp * d : nullptr;
    for (int c = lane; c < d / 4; c += 32) {
        float4 v = xr[c];
        float4 g = reinterpret_cast<const float4*>(gain)[c];
        float y[4] = {v.x * r * g.x, v.y * r * g.y, v.z * r * g.z, v.w * r * g.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            o[4 * c + i] = from_f<T>(y[i]);
            if (o2) o2[4 * c + i] = from_f<T>(y[i]);
        }
    }
}

template <typename T>
__global__ void k_merge_prep(const T* __restrict__ e, int T_alloc, const int32_t* __restrict__ pos,
                             const float* __restrict__ s, T* __restrict__ A, int B, int d, const StateHeader* sh,
                             uint64_t version, DevHeader* hdr) {
    pdl_wait();
    pdl_trigger();
    int b = blockIdx.x;
    if (b == 0 && threadIdx.x == 0 && sh) {
        if (sh->magic != STATE_MAGIC || sh->version != version) raise_flag(hdr, ERR_STATE_MISMATCH);
    }
    // e_t of this sequence's step t = pos[b] + 1 is row pos[b]; a position outside the
    // capacity the host checked means the state was changed behind the library's back
    int p = pos[b];
    if (p < 0 || p >= T_alloc) {
        if (threadIdx.x == 0) raise_flag(hdr, ERR_STATE_MISMATCH);
        p = min(max(p, 0), T_alloc - 1);
    }
    const T* er = e + ((long long)b * T_alloc + p) * d;
    T* ar = A + (long long)b * 2 * d;
    const float* sr = s + (long long)b * d;
    for (int c = threadIdx.x; c < d; c += blockDim.x) {
        ar[c] = er[c];
        ar[d + c] = from_f<T>(sr[c]);
    }
}

template <typename T>
__global__ void k_final_norm(const float* __restrict__ x, int B, int d, const float* __restrict__ gain,
                             float eps, float* __restrict__ s, T* __restrict__ hs, StateHeader* sh, int t,
                             int32_t* __restrict__ pos) {
    pdl_wait();
    pdl_trigger();
    int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    int lane = threadIdx.x & 31;
    if (warp == 0 && lane == 0 && sh) sh->t = t;
    if (warp >= B) return;
    if (lane == 0) pos[warp] += 1;                 // one more token consumed
    const float* xr = x + (long long)warp * d;
    float ss = 0.f;
    for (int c = lane; c < d; c += 32) ss += xr[c] * xr[c];
    ss = warp_sum(ss);
    float r = 1.0f / sqrtf(ss / d + eps);
    for (int c = lane; c < d; c += 32) {
        float y = xr[c] * r * gain[c];
        s[(long long)warp * d + c] = y;
        hs[(long long)warp * d + c] = from_f<T>(y);
    }
}

// One block per row.  Online (max, sum) per thread, then a block reduction.
__global__ void k_lse_gather(const float* __restrict__ logits, int B, int V, float tau,
                             const int32_t* __restrict__ tok, int tok_stride, float* logp_tok,
                             int lp_stride, float* lse_out, float* logp_full, float* score,
                             const int32_t* prompt_len, const int32_t* __restrict__ pos, DevHeader* hdr) {
    pdl_wait();
    pdl_trigger();
    int b = blockIdx.x;
    const float* z = logits + (long long)b * V;
    float m = -INFINITY, l = 0.f;
    for (int i = threadIdx.x; i < V; i += blockDim.x) {
        float v = z[i] / tau;
        if (v > m) { l = l * expf(m - v) + 1.f; m = v; }
        else l += expf(v - m);
    }
    __shared__ float sm[32], sl[32];
    int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    float mw = warp_max(m);
    l = (m == -INFINITY) ? 0.f : l * expf(m - mw);
    l = warp_sum(l);
    if (lane == 0) { sm[wid] = mw; sl[wid] = l; }
    __syncthreads();
    if (wid == 0) {
        float mm = lane < nw ? sm[lane] : -INFINITY;
        float ll = lane < nw ? sl[lane] : 0.f;
        float mx = warp_max(mm);
        ll = (mm == -INFINITY) ? 0.f : ll * expf(mm - mx);
        ll = warp_sum(ll);
        if (lane == 0) { sm[0] = mx; sl[0] = ll; }
    }
    __syncthreads();
    float lse = sm[0] + logf(sl[0]);
    if (threadIdx.x == 0) {
        if (lse_out) lse_out[b] = lse;
        if (tok) {
            int id = tok[(long long)b * tok_stride];
            if (id < 0 || id >= V) { raise_flag(hdr, ERR_BAD_TOKEN); id = 0; }
            float lp = z[id] / tau - lse;
            if (logp_tok) logp_tok[(long long)b * lp_stride] = lp;
            if (score && pos[b] >= prompt_len[b]) score[b] += lp;     // pos[b] = this step's t
        }
    }
    if (logp_full) {
        float* out = logp_full + (long long)b * V;
        for (int i = threadIdx.x; i < V; i += blockDim.x) out[i] = z[i] / tau - lse;
    }
}

// One warp per row: merge the column-tile (max, sum of exp) partials of the fused head.
__global__ void k_lse_combine(const float2* __restrict__ part, int n_tiles, const float* __restrict__ z_tok, int B,
                              int V, const int32_t* __restrict__ tok, int tok_stride, float* logp_tok, int lp_stride,
                              float* lse_out, float* score, const int32_t* prompt_len,
                              const int32_t* __restrict__ pos, DevHeader* hdr) {
    pdl_wait();
    pdl_trigger();
    const int b = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (b >= B) return;
    const float2* p = part + (long long)b * n_tiles;
    float mx = -INFINITY;
    for (int j = lane; j < n_tiles; j += 32) mx = fmaxf(mx, p[j].x);
    mx = warp_max(mx);
    float sm = 0.f;
    for (int j = lane; j < n_tiles; j += 32) sm += p[j].y * expf(p[j].x - mx);
    sm = warp_sum(sm);
    if (lane != 0) return;
    const float lse = mx + logf(sm);
    if (lse_out) lse_out[b] = lse;
    if (tok) {
        int id = tok[(long long)b * tok_stride];
        if (id < 0 || id >= V) raise_flag(hdr, ERR_BAD_TOKEN);     // the head gathered id 0
        const float lp = z_tok[b] - lse;
        if (logp_tok) logp_tok[(long long)b * lp_stride] = lp;
        if (score && pos[b] >= prompt_len[b]) score[b] += lp;          // pos[b] = this step's t
    }
}

// thread per (n, h, i < hd/2): rotate the pair (i, i + hd/2) of q and k, round q, k, v.
template <typename T>
__global__ void k_enc_qkv_layout(const float* __restrict__ qkv, int B, int Tn, int H, int hd,
                                 const float2* __restrict__ rope, T* __restrict__ planes, bool write_v) {
    pdl_wait();
    pdl_trigger();
    int half = hd / 2;
    int d = H * hd;
    long long total = (long long)B * Tn * H * half;
    long long plane = (long long)B * H * Tn * hd;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        int f = (int)(i % half);
        long long r = i / half;
        int h = (int)(r % H);
        long long n = r / H;
        int b = (int)(n / Tn), p = (int)(n % Tn);
        const float* row = qkv + n * 3 * d + h * hd;
        float2 cs = rope[(long long)p * half + f];
        long long o = (((long long)b * H + h) * Tn + p) * hd;
        float qa = row[f], qb = row[f + half];
        float ka = row[d + f], kb = row[d + f + half];
        planes[o + f] = from_f<T>(qa * cs.x - qb * cs.y);
        planes[o + f + half] = from_f<T>(qa * cs.y + qb * cs.x);
        planes[plane + o + f] = from_f<T>(ka * cs.x - kb * cs.y);
        planes[plane + o + f + half] = from_f<T>(ka * cs.y + kb * cs.x);
        if (write_v) {
            planes[2 * plane + o + f] = from_f<T>(row[2 * d + f]);
            planes[2 * plane + o + f + half] = from_f<T>(row[2 * d + f + half]);
        }
    }
}

// Encoder key/value cache of one layer, cache_l [2][B][H][T_max][hd] (keys after RoPE, both in
// the storage type, exactly as the token-parallel encoder rounds them).  Thread per
// (token n, head, pair i < hd/2) of qkv float32 [B*Tn, 3d]; token n of sequence b is position
// pos0 + n % Tn.  With q_out set (Tn = 1), the rotated query, rounded like the encoder's stored
// queries, goes to q_out [B, d] float32.
template <typename T>
__global__ void k_enc_cache_write(const float* __restrict__ qkv, int B, int Tn, int H, int hd,
                                  const float2* __restrict__ rope, int pos0, const int32_t* __restrict__ row_pos,
                                  T* __restrict__ cache_l, int T_max, float* __restrict__ q_out) {
    pdl_wait();
    pdl_trigger();
    const int half = hd / 2, d = H * hd;
    const long long total = (long long)B * Tn * H * half;
    const long long plane = (long long)B * H * T_max * hd;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int f = (int)(i % half);
        const long long r = i / half;
        const int h = (int)(r % H);
        const long long n = r / H;
        const int b = (int)(n / Tn);
        const int p = row_pos ? min(max(row_pos[b], 0), T_max - 1) : pos0 + (int)(n % Tn);
        const float* row = qkv + n * 3 * d + h * hd;
        const float2 cs = rope[(long long)p * half + f];
        const long long o = (((long long)b * H + h) * T_max + p) * hd;
        const float ka = row[d + f], kb = row[d + f + half];
        cache_l[o + f] = from_f<T>(ka * cs.x - kb * cs.y);
        cache_l[o + f + half] = from_f<T>(ka * cs.y + kb * cs.x);
        cache_l[plane + o + f] = from_f<T>(row[2 * d + f]);
        cache_l[plane + o + f + half] = from_f<T>(row[2 * d + f + half]);
        if (q_out) {
            const float qa = row[f], qb = row[f + half];
            float* qo = q_out + (long long)b * d + h * hd;
            qo[f] = round_to<T>(qa * cs.x - qb * cs.y);
            qo[f + half] = round_to<T>(qa * cs.y + qb * cs.x);
        }
    }
}

template <typename T>
__global__ void k_mem_layout(const float* __restrict__ kv, int B, int Tn, int T_alloc, int H, int hd,
                             T* __restrict__ Mg, const int32_t* __restrict__ row_pos) {
    pdl_wait();
    pdl_trigger();
    int d = H * hd;
    long long total = (long long)B * Tn * 2 * d;
    long long plane = (long long)B * H * T_alloc * hd;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        int c = (int)(i % (2 * d));
        long long n = i / (2 * d);
        int b = (int)(n / Tn);
        int p = row_pos ? min(max(row_pos[b], 0), T_alloc - 1) : (int)(n % Tn);
        int kvsel = c / d, h = (c % d) / hd, x = c % hd;
        Mg[kvsel * plane + (((long long)b * H + h) * T_alloc + p) * hd + x] = from_f<T>(kv[i]);
    }
}

__global__ void k_state_init(const float* __restrict__ s_star, int B, int d, float* __restrict__ s,
                             StateHeader* sh, uint64_t version, int32_t* __restrict__ pos, int row) {
    pdl_wait();
    pdl_trigger();
    // every row, or only row `row` (>= 0) of a batch state
    const long long n = row >= 0 ? d : (long long)B * d;
    float* s0 = row >= 0 ? s + (long long)row * d : s;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x)
        s0[i] = s_star[i % d];
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < (row >= 0 ? 1 : B);
         i += (long long)gridDim.x * blockDim.x)
        pos[row >= 0 ? row : i] = 0;
    if (row >= 0) return;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        sh->magic = STATE_MAGIC;
        sh->t = 0;
        sh->version = version;
        sh->B = B;
    }
}

inline unsigned grid_for(long long n, int threads) {
    long long g = (n + threads - 1) / threads;
    return (unsigned)(g > 148LL * 64 ? 148LL * 64 : (g < 1 ? 1 : g));
}


}  // namespace

template <typename T>
cudaError_t launch_pack_rows(Launch L, const float* src, T* dst, int rows, int cols, int dst_ld,
                             int row_mult, int row_off, int col_off) {
    return launch_k(L, k_pack_rows<T>, grid_for((long long)rows * cols, 256), 256, 0, src, dst, rows, cols, dst_ld,
                    row_mult, row_off, col_off);
}

cudaError_t launch_rope_table(Launch L, float2* table, int max_pos, int head_dim, float base) {
    int half = head_dim / 2;
    return launch_k(L, k_rope_table, grid_for((long long)max_pos * half, 256), 256, 0, table, max_pos, half, head_dim,
                    (double)base);
}

template <typename T>
cudaError_t launch_embed(Launch L, const int32_t* tok, int N, const T* embed, int V, int d, float* h,
                         DevHeader* hdr, int tok_stride) {
    return launch_k(L, k_embed<T>, N, 128, 0, tok, tok_stride, N, embed, V, d, h, hdr);
}

template <typename T>
cudaError_t launch_rmsnorm(Launch L, const float* x, int N, int d, const float* gain, float eps, T* out,
                           int out_ld, int rows_per_seq, int out_rows_per_seq, T* out2, const int32_t* row_pos) {
    return launch_k(L, k_rmsnorm<T>, cdiv(N, 8), 256, 0, x, N, d, gain, eps, out, out_ld, rows_per_seq,
                    out_rows_per_seq, out2, row_pos);
}

template <typename T>
cudaError_t launch_merge_prep(Launch L, const T* e, int T_alloc, const int32_t* pos, const float* s, T* A, int B,
                              int d, const StateHeader* sh, uint64_t version, DevHeader* hdr) {
    return launch_k(L, k_merge_prep<T>, B, 256, 0, e, T_alloc, pos, s, A, B, d, sh, version, hdr);
}

template <typename T>
cudaError_t launch_final_norm(Launch L, const float* x, int B, int d, const float* gain, float eps,
                              float* s, T* hs, StateHeader* sh, int t, int32_t* pos) {
    return launch_k(L, k_final_norm<T>, cdiv(B, 8), 256, 0, x, B, d, gain, eps, s, hs, sh, t, pos);
}

cudaError_t launch_lse_gather(Launch L, const float* logits, int B, int V, float tau, const int32_t* tok,
                              int tok_stride, float* logp_tok, int lp_stride, float* lse,
                              float* logp_full, float* score, const int32_t* prompt_len, const int32_t* pos,
                              DevHeader* hdr) {
    return launch_k(L, k_lse_gather, B, 512, 0, logits, B, V, tau, tok, tok_stride, logp_tok, lp_stride, lse,
                    logp_full, score, prompt_len, pos, hdr);
}

cudaError_t launch_lse_combine(Launch L, const float2* part, int n_tiles, const float* z_tok, int B, int V,
                               const int32_t* tok, int tok_stride, float* logp_tok, int lp_stride, float* lse,
                               float* score, const int32_t* prompt_len, const int32_t* pos, DevHeader* hdr) {
    return launch_k(L, k_lse_combine, cdiv(B, 8), 256, 0, part, n_tiles, z_tok, B, V, tok, tok_stride, logp_tok,
                    lp_stride, lse, score, prompt_len, pos, hdr);
}

template <typename T>
cudaError_t launch_enc_qkv_layout(Launch L, const float* qkv, int B, int Tn, int H, int hd,
                                  const float2* rope, T* planes, bool write_v) {
    return launch_k(L, k_enc_qkv_layout<T>, grid_for((long long)B * Tn * H * (hd / 2), 256), 256, 0, qkv, B, Tn, H,
                    hd, rope, planes, write_v);
}

template <typename T>
cudaError_t launch_mem_layout(Launch L, const float* kv, int B, int Tn, int T_alloc, int H, int hd, T* Mg,
                              const int32_t* row_pos) {
    return launch_k(L, k_mem_layout<T>, grid_for((long long)B * Tn * 2 * H * hd, 256), 256, 0, kv, B, Tn, T_alloc,
                    H, hd, Mg, row_pos);
}

template <typename T>
cudaError_t launch_enc_cache_write(Launch L, const float* qkv, int B, int Tn, int H, int hd, const float2* rope,
                                   int pos0, const int32_t* row_pos, T* cache_l, int T_max, float* q_out) {
    return launch_k(L, k_enc_cache_write<T>, grid_for((long long)B * Tn * H * (hd / 2), 256), 256, 0, qkv, B, Tn, H,
                    hd, rope, pos0, row_pos, cache_l, T_max, q_out);
}

cudaError_t launch_state_init(Launch L, const float* s_star, int B, int d, float* s, StateHeader* sh,
                              uint64_t version, int32_t* pos, int row) {
    return launch_k(L, k_state_init, grid_for((long long)(row >= 0 ? 1 : B) * d, 256), 256, 0, s_star, B, d, s, sh,
                    version, pos, row);
}

#define RLT_INST(T)                                                                                   \
    template cudaError_t launch_pack_rows<T>(Launch, const float*, T*, int, int, int, int, int, int); \
    template cudaError_t launch_embed<T>(Launch, const int32_t*, int, const T*, int, int, float*,     \
                                         DevHeader*, int);                                            \
    template cudaError_t launch_rmsnorm<T>(Launch, const float*, int, int, const float*, float, T*,   \
                                           int, int, int, T*, const int32_t*);                        \
    template cudaError_t launch_merge_prep<T>(Launch, const T*, int, const int32_t*, const float*, T*, \
                                              int, int, const StateHeader*, uint64_t, DevHeader*);    \
    template cudaError_t launch_final_norm<T>(Launch, const float*, int, int, const float*, float,    \
                                              float*, T*, StateHeader*, int, int32_t*);               \
    template cudaError_t launch_enc_qkv_layout<T>(Launch, const float*, int, int, int, int,           \
                                                  const float2*, T*, bool);                           \
    template cudaError_t launch_mem_layout<T>(Launch, const float*, int, int, int, int, int, T*,      \
                                              const int32_t*);                                        \
    template cudaError_t launch_enc_cache_write<T>(Launch, const float*, int, int, int, int, const float2*, int, \
                                                   const int32_t*, T*, int, float*);
RLT_INST(float)
RLT_INST(bf16)
#undef RLT_INST

}  // namespace rlt
