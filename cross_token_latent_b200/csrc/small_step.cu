// The whole decoder step of a small model in one launch: one CTA per sequence.
//
// Sequences are independent ([news] model-hardware principle), so a step needs no
// communication between them.  For models whose weights stay resident in L2 (d <= 256,
// F <= 1024, V <= 8192: the tiny and small workloads), one CTA of 512 threads runs every part
// of one sequence's transition back to back -- the gated merge, each layer's SWA over its ring,
// cross-attention over its M_{<=t}, SwiGLU FFN, the final norm and the head with its
// log-sum-exp -- with __syncthreads between the phases.  That replaces ~10 kernel launches per
// layer (each paying its launch, prologue and drain on the GPU) by one launch per step.
//
// Arithmetic follows the storage contract exactly as the oracle states it: the sublayer norm
// is computed in float32 and its output rounded to the storage type before the projection;
// attention outputs, SiLU(g) * u and s fed to the merge and the head are rounded likewise;
// decoder queries, softmax, the residual stream, s_t and log-probabilities stay float32.
// Projections are warp-per-output-row dot products over rows of W read from L2 (16-byte
// loads) against the input vector in shared memory.  Attention gives every head
// SS_WARPS / n_heads warps, one key per lane, whose online-softmax states are merged through
// shared memory (head_dim 16 or 32).
#include "kernels.cuh"

namespace rlt {

namespace {

constexpr int SS_THREADS = 512;
constexpr int SS_WARPS = SS_THREADS / 32;
constexpr int SS_MAX_D = 256, SS_MAX_F = 1024, SS_MAX_V = 8192;

// y[n] = sum_k W[n, k] x[k] for n < N (W row-major [N, K] in storage type, x float in shared
// memory).  A row is split over a group of lpr lanes (lpr = the power of two <= K/8 up to 32,
// 16-byte pieces each), a warp works on 32/lpr rows per pass and GV_U passes at once, so that
// several independent row loads are in flight per lane; the group reduces by shuffles.
template <typename T>
__device__ __forceinline__ void gemv_rows(const T* __restrict__ W, int N, int K, const float* x, float* y) {
    constexpr int EPL = Vec16<T>::N;
    constexpr int U = 4;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nv = K / EPL;
    int lpr = 32;
    while (lpr > 1 && lpr > nv) lpr >>= 1;
    const int rpp = 32 / lpr, sub = lane / lpr, li = lane % lpr;
    for (int base = warp * rpp * U; base < N; base += SS_WARPS * rpp * U) {
        float acc[U];
#pragma unroll
        for (int u = 0; u < U; ++u) acc[u] = 0.f;
        for (int v = li; v < nv; v += lpr) {
            uint4 wv[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int n = base + u * rpp + sub;
                wv[u] = n < N ? __ldg(reinterpret_cast<const uint4*>(W + (size_t)n * K) + v) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                float w[EPL];
                Vec16<T>::unpack(wv[u], w);
#pragma unroll
                for (int i = 0; i < EPL; ++i) acc[u] = fmaf(w[i], x[v * EPL + i], acc[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float a = acc[u];
            for (int o = lpr / 2; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
            const int n = base + u * rpp + sub;
            if (li == 0 && n < N) y[n] = a;
        }
    }
}

// RMSNorm(x) * g rounded to the storage type (as float) into h; every thread returns after
// the block-wide reduction (uses red[SS_WARPS]).
template <typename T>
__device__ __forceinline__ void norm_round(const float* x, int d, const float* __restrict__ g, float eps, float* h,
                                           float* red) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float ss = 0.f;
    for (int c = threadIdx.x; c < d; c += SS_THREADS) ss += x[c] * x[c];
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    float tot = 0.f;
    for (int w = 0; w < SS_WARPS; ++w) tot += red[w];
    const float r = 1.0f / sqrtf(tot / d + eps);
    for (int c = threadIdx.x; c < d; c += SS_THREADS) h[c] = round_to<T>(x[c] * r * g[c]);
    __syncthreads();
}

// Partial softmax state of one warp over its keys: lanes take keys j = j0 + lane, j0 + lane +
// stride, ... (< n) of K, V (storage type, row stride HD), q float (already scaled by
// log2(e)/sqrt(hd)); optionally one extra key/value in float (the current token) folded in by
// lane 0.  On return every lane holds the warp's (m, l, acc).
template <typename T, int HD>
__device__ __forceinline__ void warp_partial(const float* q, const T* __restrict__ K, const T* __restrict__ V, int j0,
                                             int n, int stride, const float* kx, const float* vx, float& m, float& l,
                                             float* acc) {
    const int lane = threadIdx.x & 31;
    constexpr int EPL = Vec16<T>::N;
    m = -1e30f;
    l = 0.f;
#pragma unroll
    for (int i = 0; i < HD; ++i) acc[i] = 0.f;
    auto fold = [&](float s, const float* vrow) {
        const float mx = fmaxf(m, s);
        const float c = exp2f(m - mx), p = exp2f(s - mx);
        l = l * c + p;
#pragma unroll
        for (int i = 0; i < HD; ++i) acc[i] = acc[i] * c + p * vrow[i];
        m = mx;
    };
    for (int j = j0 + lane; j < n; j += stride) {
        float r[HD];
#pragma unroll
        for (int v = 0; v < HD / EPL; ++v) Vec16<T>::unpack(ld16(K + (size_t)j * HD + v * EPL), r + v * EPL);
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < HD; ++i) s = fmaf(q[i], r[i], s);
#pragma unroll
        for (int v = 0; v < HD / EPL; ++v) Vec16<T>::unpack(ld16(V + (size_t)j * HD + v * EPL), r + v * EPL);
        fold(s, r);
    }
    if (kx && lane == 0) {
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < HD; ++i) s = fmaf(q[i], kx[i], s);
        fold(s, vx);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, m, o), lo = __shfl_xor_sync(0xffffffffu, l, o);
        const float mx = fmaxf(m, mo);
        const float c1 = exp2f(m - mx), c2 = exp2f(mo - mx);
        l = l * c1 + lo * c2;
#pragma unroll
        for (int i = 0; i < HD; ++i) acc[i] = acc[i] * c1 + __shfl_xor_sync(0xffffffffu, acc[i], o) * c2;
        m = mx;
    }
}

// Shared scratch of the per-head attention: each warp's partial state.
template <int HD>
struct AttnScratch {
    float m[SS_WARPS], l[SS_WARPS];
    float acc[SS_WARPS][HD];
};

// Merge the partial states of head hh's wph warps (warps hh*wph .. hh*wph+wph-1) and write the
// normalised output rounded to the storage type into out[hh*HD ..].  Called by the first warp
// of the head after a __syncthreads.
template <typename T, int HD>
__device__ __forceinline__ void merge_head(const AttnScratch<HD>& sc, int hh, int wph, float* out) {
    const int lane = threadIdx.x & 31;
    float mx = -1e30f;
    for (int w = 0; w < wph; ++w) mx = fmaxf(mx, sc.m[hh * wph + w]);
    float L = 0.f;
    for (int w = 0; w < wph; ++w) L += sc.l[hh * wph + w] * exp2f(sc.m[hh * wph + w] - mx);
    for (int i = lane; i < HD; i += 32) {
        float a = 0.f;
        for (int w = 0; w < wph; ++w) a += sc.acc[hh * wph + w][i] * exp2f(sc.m[hh * wph + w] - mx);
        out[hh * HD + i] = round_to<T>(a / L);
    }
}

template <typename T, int HD>
__global__ void __launch_bounds__(SS_THREADS) k_small_step(SmallStepArgs a) {
    __shared__ float x[SS_MAX_D];
    __shared__ float h[2 * SS_MAX_D > SS_MAX_F ? 2 * SS_MAX_D : SS_MAX_F];
    __shared__ float y[2 * SS_MAX_F > 3 * SS_MAX_D ? 2 * SS_MAX_F : 3 * SS_MAX_D];
    __shared__ float att[SS_MAX_D];
    __shared__ float red[SS_WARPS];
    __shared__ AttnScratch<HD> sc;
    extern __shared__ float logits[];                // V floats
    pdl_wait();
    pdl_trigger();
    const int b = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int d = a.d, H = a.H, F = a.F, V = a.V, W = a.W, half = HD / 2;
    const int wph = SS_WARPS / H;                    // warps per head (H <= 16)
    const float qscale = 1.4426950408889634f / sqrtf((float)HD);
    const DecWeights& w = a.w;
    auto mat = [](const void* p) { return static_cast<const T*>(p); };

    if (b == 0 && threadIdx.x == 0 && a.sh) {
        if (a.sh->magic != STATE_MAGIC || a.sh->version != a.version) raise_flag(a.hdr, ERR_STATE_MISMATCH);
        a.sh->t = a.t_host;
    }
    int p = a.pos[b];
    if (p < 0 || p >= a.T_alloc) {
        if (threadIdx.x == 0) raise_flag(a.hdr, ERR_STATE_MISMATCH);
        p = min(max(p, 0), a.T_alloc - 1);
    }
    const int t = p + 1;
    const float2* rope_row = a.rope + (size_t)p * half;

    // gated merge: h = [e_t | bf16(s_{t-1})], rows 2j / 2j+1 of W_m are gate_j / feedback_j
    const T* er = static_cast<const T*>(a.e) + ((size_t)b * a.T_alloc + p) * d;
    float* s = a.s + (size_t)b * d;
    for (int c = threadIdx.x; c < d; c += SS_THREADS) {
        h[c] = to_f(er[c]);
        h[d + c] = round_to<T>(s[c]);
    }
    __syncthreads();
    gemv_rows<T>(mat(w.merge), 2 * d, 2 * d, h, y);
    __syncthreads();
    for (int c = threadIdx.x; c < d; c += SS_THREADS) x[c] = h[c] + sigmoidf_(y[2 * c] + w.merge_b[c]) * y[2 * c + 1];
    __syncthreads();

    for (int l = 0; l < a.L; ++l) {
        // ---- sliding-window self-attention (encoder layer l's weights)
        norm_round<T>(x, d, w.attn_norm[l], a.eps, h, red);
        gemv_rows<T>(mat(w.wqkv[l]), 3 * d, d, h, y);
        __syncthreads();
        T* ring_l = static_cast<T*>(a.ring) + (size_t)l * a.ring_layer;
        {
            // head hh = warp / wph; its wph warps split the cached entries, the first of them
            // also attends to the current token and later writes it into the ring
            const int hh = warp / wph, sub = warp % wph;
            float q[HD], k[HD], v[HD], mm, ll, acc[HD];
            T* Kr = nullptr;
            T* Vr = nullptr;
            if (hh < H) {
#pragma unroll
                for (int i = 0; i < HD; ++i) {
                    const int cp = i < half ? i + half : i - half;
                    const float2 cs = rope_row[i % half];
                    const float qa = y[hh * HD + i], qp = y[hh * HD + cp];
                    const float ka = y[d + hh * HD + i], kp = y[d + hh * HD + cp];
                    q[i] = (i < half ? qa * cs.x - qp * cs.y : qp * cs.y + qa * cs.x) * qscale;
                    k[i] = round_to<T>(i < half ? ka * cs.x - kp * cs.y : kp * cs.y + ka * cs.x);
                    v[i] = round_to<T>(y[2 * d + hh * HD + i]);
                }
                Kr = ring_l + (((size_t)b * 2 + 0) * H + hh) * (size_t)(W - 1) * HD;
                Vr = ring_l + (((size_t)b * 2 + 1) * H + hh) * (size_t)(W - 1) * HD;
                const int n = W > 1 ? min(t - 1, W - 1) : 0;
                warp_partial<T, HD>(q, Kr, Vr, sub * 32, n, wph * 32, sub == 0 ? k : nullptr, v, mm, ll, acc);
                if (lane == 0) { sc.m[warp] = mm; sc.l[warp] = ll; }
                for (int i = lane; i < HD; i += 32) sc.acc[warp][i] = acc[i];
            }
            __syncthreads();                            // every warp has read its ring entries
            if (hh < H && sub == 0) {
                merge_head<T, HD>(sc, hh, wph, att);
                if (W > 1 && lane == 0) {
                    const int slot = (t - 1) % (W - 1);
#pragma unroll
                    for (int i = 0; i < HD; ++i) {
                        Kr[(size_t)slot * HD + i] = from_f<T>(k[i]);
                        Vr[(size_t)slot * HD + i] = from_f<T>(v[i]);
                    }
                }
            }
        }
        __syncthreads();
        gemv_rows<T>(mat(w.wo[l]), d, d, att, y);
        __syncthreads();
        for (int c = threadIdx.x; c < d; c += SS_THREADS) x[c] += y[c];
        __syncthreads();
        // ---- cross-attention to M_{<=t} (no rotary embedding)
        norm_round<T>(x, d, w.xattn_norm[l], a.eps, h, red);
        gemv_rows<T>(mat(w.wqc[l]), d, d, h, y);
        __syncthreads();
        const T* Mg = static_cast<const T*>(a.M) + (a.G == 1 ? 0 : (size_t)l * a.group_elems);
        {
            const int hh = warp / wph, sub = warp % wph;
            if (hh < H) {
                float q[HD], mm, ll, acc[HD];
#pragma unroll
                for (int i = 0; i < HD; ++i) q[i] = y[hh * HD + i] * qscale;
                const T* Km = Mg + ((size_t)b * H + hh) * (size_t)a.T_alloc * HD;
                warp_partial<T, HD>(q, Km, Km + a.plane, sub * 32, t, wph * 32, nullptr, nullptr, mm, ll, acc);
                if (lane == 0) { sc.m[warp] = mm; sc.l[warp] = ll; }
                for (int i = lane; i < HD; i += 32) sc.acc[warp][i] = acc[i];
            }
            __syncthreads();
            if (hh < H && sub == 0) merge_head<T, HD>(sc, hh, wph, att);
        }
        __syncthreads();
        gemv_rows<T>(mat(w.woc[l]), d, d, att, y);
        __syncthreads();
        for (int c = threadIdx.x; c < d; c += SS_THREADS) x[c] += y[c];
        __syncthreads();
        // ---- SwiGLU FFN (rows 2j / 2j+1 of W_gu are gate_j / up_j)
        norm_round<T>(x, d, w.ffn_norm[l], a.eps, h, red);
        gemv_rows<T>(mat(w.wgu[l]), 2 * F, d, h, y);
        __syncthreads();
        for (int c = threadIdx.x; c < F; c += SS_THREADS) h[c] = round_to<T>(siluf_(y[2 * c]) * y[2 * c + 1]);
        __syncthreads();
        gemv_rows<T>(mat(w.wdown[l]), d, F, h, y);
        __syncthreads();
        for (int c = threadIdx.x; c < d; c += SS_THREADS) x[c] += y[c];
        __syncthreads();
    }

    // split: s_t = RMSNorm(x) (float32, the new state) and the head from bf16(s_t)
    {
        float ss = 0.f;
        for (int c = threadIdx.x; c < d; c += SS_THREADS) ss += x[c] * x[c];
        ss = warp_sum(ss);
        if (lane == 0) red[warp] = ss;
        __syncthreads();
        float tot = 0.f;
        for (int ww = 0; ww < SS_WARPS; ++ww) tot += red[ww];
        const float r = 1.0f / sqrtf(tot / d + a.eps);
        for (int c = threadIdx.x; c < d; c += SS_THREADS) {
            const float v = x[c] * r * w.dec_norm[c];
            s[c] = v;
            h[c] = round_to<T>(v);
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) a.pos[b] = p + 1;
    if (!a.head) return;
    gemv_rows<T>(mat(w.unembed), V, d, h, logits);
    __syncthreads();
    // log-sum-exp of z = logits / tau
    float m = -INFINITY;
    for (int i = threadIdx.x; i < V; i += SS_THREADS) m = fmaxf(m, logits[i] / a.tau);
    m = warp_max(m);
    if (lane == 0) red[warp] = m;
    __syncthreads();
    float mx = -INFINITY;
    for (int ww = 0; ww < SS_WARPS; ++ww) mx = fmaxf(mx, red[ww]);
    __syncthreads();
    float sum = 0.f;
    for (int i = threadIdx.x; i < V; i += SS_THREADS) sum += expf(logits[i] / a.tau - mx);
    sum = warp_sum(sum);
    if (lane == 0) red[warp] = sum;
    __syncthreads();
    float tot = 0.f;
    for (int ww = 0; ww < SS_WARPS; ++ww) tot += red[ww];
    const float lse = mx + logf(tot);
    if (threadIdx.x == 0) {
        if (a.lse) a.lse[b] = lse;
        if (a.tok) {
            int id = a.tok[(size_t)b * a.tok_stride];
            if (id < 0 || id >= V) { raise_flag(a.hdr, ERR_BAD_TOKEN); id = 0; }
            const float lp = logits[id] / a.tau - lse;
            if (a.logp_tok) a.logp_tok[(size_t)b * a.lp_stride] = lp;
            if (a.score && t >= a.prompt_len[b]) a.score[b] += lp;
        }
    }
    if (a.logp_full)
        for (int i = threadIdx.x; i < V; i += SS_THREADS) a.logp_full[(size_t)b * V + i] = logits[i] / a.tau - lse;
}

}  // namespace

bool small_step_supported(int d, int F, int V, int hd, int L) {
    return d <= SS_MAX_D && F <= SS_MAX_F && V <= SS_MAX_V && L <= SS_MAX_LAYERS && d % 8 == 0 && d / hd <= SS_WARPS &&
           F % 8 == 0 && (hd == 16 || hd == 32);
}

template <typename T>
cudaError_t launch_small_step(Launch L, const SmallStepArgs& a, int hd) {
    const size_t smem = (size_t)a.V * 4;
    switch (hd) {
        case 16: return launch_k(L, k_small_step<T, 16>, (unsigned)a.B, SS_THREADS, smem, a);
        case 32: return launch_k(L, k_small_step<T, 32>, (unsigned)a.B, SS_THREADS, smem, a);
    }
    return cudaErrorInvalidValue;
}

template cudaError_t launch_small_step<float>(Launch, const SmallStepArgs&, int);
template cudaError_t launch_small_step<bf16>(Launch, const SmallStepArgs&, int);

}  // namespace rlt
