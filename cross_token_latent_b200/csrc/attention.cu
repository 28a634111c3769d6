// Warp-level online-softmax attention of the RLT path.
//
// One warp owns one (sequence, head[, key chunk]) work item.  Lanes are grouped so that
// LPK lanes hold one key row with 16-byte loads (LPK = head_dim * sizeof(T) / 16); the
// KPI = 32 / LPK groups walk interleaved keys, keep their own running (max, sum, acc)
// and are merged by shuffles at the end.  Keys and values are streamed with coalesced
// 16-byte loads, several rounds in flight per lane.  Used for
//   - decoder sliding-window self-attention over the ring cache plus the current token,
//   - decoder cross-attention over the causal encoder memory M_{<=t} (split along keys
//     when there are too few (sequence, head) pairs to fill the GPU),
//   - the encoder's causal self-attention (one query per warp).
#include "kernels.cuh"

namespace rlt {

namespace {

constexpr float LOG2E = 1.4426950408889634f;
constexpr float NEG_BIG = -1e30f;
constexpr int WARPS = 4;

template <typename T, int HD>
struct Geom {
    static constexpr int EPL = 16 / (int)sizeof(T);   // elements per lane
    static constexpr int LPK = HD / EPL;               // lanes per key row
    static constexpr int KPI = 32 / LPK;               // keys per warp round
    static_assert(LPK >= 1 && LPK <= 32 && 32 % LPK == 0, "head_dim not supported");
};

template <int LPK>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
    for (int o = LPK / 2; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// One round of the key loop: KPI * U keys starting at `base`, one 16-byte piece of a K row and
// of a V row per lane and key (zeros past n).
template <typename T, int HD, int U, bool STREAM>
__device__ __forceinline__ void load_round(const T* __restrict__ K, const T* __restrict__ V, int n, int base, int g,
                                           int li, uint4* kr, uint4* vr) {
    using G = Geom<T, HD>;
#pragma unroll
    for (int u = 0; u < U; ++u) {
        int j = base + u * G::KPI + g;
        if (j < n) {
            const T* kp = K + (long long)j * HD + li * G::EPL;
            const T* vp = V + (long long)j * HD + li * G::EPL;
            kr[u] = STREAM ? ld16_stream(kp) : ld16(kp);
            vr[u] = STREAM ? ld16_stream(vp) : ld16(vp);
        } else {
            kr[u] = make_uint4(0, 0, 0, 0);
            vr[u] = make_uint4(0, 0, 0, 0);
        }
    }
}

// Fold one loaded round into this lane group's running softmax (m, l, acc).
template <typename T, int HD, int U>
__device__ __forceinline__ void consume_round(const float* q, int n, int base, int g, const uint4* kr, const uint4* vr,
                                              float& m, float& l, float* acc) {
    using G = Geom<T, HD>;
    constexpr int EPL = G::EPL, LPK = G::LPK, KPI = G::KPI;
    float s[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        float kf[EPL];
        Vec16<T>::unpack(kr[u], kf);
        float dot = 0.f;
#pragma unroll
        for (int i = 0; i < EPL; ++i) dot = fmaf(q[i], kf[i], dot);
        dot = group_sum<LPK>(dot);
        s[u] = (base + u * KPI + g < n) ? dot : NEG_BIG;
    }
    float mx = m;
#pragma unroll
    for (int u = 0; u < U; ++u) mx = fmaxf(mx, s[u]);
    float corr = exp2f(m - mx);
    l *= corr;
#pragma unroll
    for (int i = 0; i < EPL; ++i) acc[i] *= corr;
#pragma unroll
    for (int u = 0; u < U; ++u) {
        float p = (base + u * KPI + g < n) ? exp2f(s[u] - mx) : 0.f;
        l += p;
        float vf[EPL];
        Vec16<T>::unpack(vr[u], vf);
#pragma unroll
        for (int i = 0; i < EPL; ++i) acc[i] = fmaf(p, vf[i], acc[i]);
    }
    m = mx;
}

// Accumulate keys [base0, n) of K/V (row stride HD) into this lane group's running softmax.
// q is pre-scaled by log2(e)/sqrt(hd).  n must be warp-uniform.
template <typename T, int HD, int U, bool STREAM>
__device__ __forceinline__ void attend(const float* q, const T* __restrict__ K, const T* __restrict__ V,
                                       int n, int g, int li, float& m, float& l, float* acc, int base0 = 0) {
    using G = Geom<T, HD>;
    for (int base = base0; base < n; base += G::KPI * U) {
        uint4 kr[U], vr[U];
        load_round<T, HD, U, STREAM>(K, V, n, base, g, li, kr, vr);
        consume_round<T, HD, U>(q, n, base, g, kr, vr, m, l, acc);
    }
}

// Merge the KPI lane groups' running softmax states; afterwards every group holds the total.
template <typename T, int HD>
__device__ __forceinline__ void merge_groups(float& m, float& l, float* acc) {
    using G = Geom<T, HD>;
#pragma unroll
    for (int o = G::LPK; o < 32; o <<= 1) {
        float mo = __shfl_xor_sync(0xffffffffu, m, o);
        float lo = __shfl_xor_sync(0xffffffffu, l, o);
        float mx = fmaxf(m, mo);
        float c1 = exp2f(m - mx), c2 = exp2f(mo - mx);
        l = l * c1 + lo * c2;
#pragma unroll
        for (int i = 0; i < G::EPL; ++i) {
            float ao = __shfl_xor_sync(0xffffffffu, acc[i], o);
            acc[i] = acc[i] * c1 + ao * c2;
        }
        m = mx;
    }
}

// One CTA of SWA_WARPS warps per (sequence, head) and key split.  Every warp computes q (RoPE
// at position t-1); the n = min(t-1, W-1) cached entries are cut into n_splits contiguous
// ranges of ring slots, one per CTA, and warp w of a CTA streams a contiguous share of its
// range; the warps' partial softmax states are merged through shared memory.  Split 0 also
// attends to the current token (k_t, v_t rounded to the storage type).  The CTA whose range
// holds ring slot (t-1) mod (W-1) (split 0 while the ring is not yet full) stores k_t, v_t
// there after its warps have read the slot's old entry -- token t-W+1, still in the window.
// With one split the CTA writes the normalised output; with several, each writes its
// unnormalised partial (acc, max, sum) and k_attn_combine merges them.
constexpr int SWA_WARPS = 4;

template <typename T, int HD>
__global__ void __launch_bounds__(SWA_WARPS * 32, 6) k_swa_decode(const float* __restrict__ qkv,
                                                                  const float2* __restrict__ rope,
                                                                  T* __restrict__ ring, T* __restrict__ o,
                                                                  int B, int H, int W, const int32_t* __restrict__ pos,
                                                                  int max_t, int n_splits, float* __restrict__ part,
                                                                  float qscale) {
    using G = Geom<T, HD>;
    constexpr int EPL = G::EPL, LPK = G::LPK;
    __shared__ float sm_m[SWA_WARPS], sm_l[SWA_WARPS];
    __shared__ __align__(16) float sm_acc[SWA_WARPS][HD];
    __shared__ __align__(16) uint4 sm_kv[2][LPK];      // current k_t, v_t in storage type
    pdl_wait();
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane / LPK, li = lane % LPK;
    const int d = H * HD, half = HD / 2;
    // one (sequence, head, split) work item per iteration; the grid is at most one item per CTA
    // and may be capped below that (then each CTA takes items blockIdx.x, blockIdx.x +
    // gridDim.x, ...)
    for (int wi = blockIdx.x; wi < B * H * n_splits; wi += gridDim.x) {
        const int item = wi / n_splits, sp = wi % n_splits;
        const int b = item / H, h = item % H;
        // this sequence's step t: it has consumed pos[b] tokens (clamped to the bound the host
        // checked, so that a corrupt state cannot address outside the rotary table)
        const int t = min(max(pos[b] + 1, 1), max_t);
        const float2* rope_row = rope + (long long)(t - 1) * half;
        const float* row = qkv + (long long)b * 3 * d + h * HD;
        // this split's range of ring slots, and this warp's share of it; the warp's first round
        // of loads is issued before q is formed, so the ring's memory latency overlaps the q /
        // RoPE loads instead of following them
        T* Kr = nullptr;
        T* Vr = nullptr;
        int j0 = 0, nj = 0, s0 = 0, s1 = 0, slot = 0;
        bool writer = false;
        if (W > 1) {
            Kr = ring + (((long long)b * 2 + 0) * H + h) * (long long)(W - 1) * HD;
            Vr = ring + (((long long)b * 2 + 1) * H + h) * (long long)(W - 1) * HD;
            const int n = min(t - 1, W - 1);
            const int per_split = (n + n_splits - 1) / n_splits;
            s0 = min(n, sp * per_split);
            s1 = min(n, s0 + per_split);
            const int per = (s1 - s0 + SWA_WARPS - 1) / SWA_WARPS;
            j0 = min(s1, s0 + warp * per);
            nj = min(s1, j0 + per) - j0;
            slot = (t - 1) % (W - 1);
            writer = slot < n ? (slot >= s0 && slot < s1) : sp == 0;
        }
        constexpr int SWA_U = 4;
        uint4 kr0[SWA_U], vr0[SWA_U];
        load_round<T, HD, SWA_U, true>(Kr + (long long)j0 * HD, Vr + (long long)j0 * HD, nj, 0, g, li, kr0, vr0);
        float q[EPL];
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            int c = li * EPL + i;
            int cp = c < half ? c + half : c - half;
            float2 cs = rope_row[c % half];
            float qa = row[c], qp = row[cp];
            q[i] = (c < half ? qa * cs.x - qp * cs.y : qp * cs.y + qa * cs.x) * qscale;
        }
        float m = NEG_BIG, l = 0.f, acc[EPL];
#pragma unroll
        for (int i = 0; i < EPL; ++i) acc[i] = 0.f;
        if (warp == 0 && (sp == 0 || writer)) {
            // the current token: k_t (rotated) and v_t rounded to the storage type, as cached
            float k[EPL], v[EPL];
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                int c = li * EPL + i;
                int cp = c < half ? c + half : c - half;
                float2 cs = rope_row[c % half];
                float ka = row[d + c], kp = row[d + cp];
                k[i] = round_to<T>(c < half ? ka * cs.x - kp * cs.y : kp * cs.y + ka * cs.x);
                v[i] = round_to<T>(row[2 * d + c]);
            }
            if (sp == 0) {
                float sc = 0.f;
#pragma unroll
                for (int i = 0; i < EPL; ++i) sc = fmaf(q[i], k[i], sc);
                sc = group_sum<LPK>(sc);
                if (g == 0) {
                    m = sc; l = 1.f;
#pragma unroll
                    for (int i = 0; i < EPL; ++i) acc[i] = v[i];
                }
            }
            if (g == 0) {
                sm_kv[0][li] = Vec16<T>::pack(k);
                sm_kv[1][li] = Vec16<T>::pack(v);
            }
        }
        if (nj > 0) {
            consume_round<T, HD, SWA_U>(q, nj, 0, g, kr0, vr0, m, l, acc);
            attend<T, HD, SWA_U, true>(q, Kr + (long long)j0 * HD, Vr + (long long)j0 * HD, nj, g, li, m, l, acc,
                                       Geom<T, HD>::KPI * SWA_U);
        }
        merge_groups<T, HD>(m, l, acc);
        if (g == 0) {
#pragma unroll
            for (int i = 0; i < EPL; ++i) sm_acc[warp][li * EPL + i] = acc[i];
            if (li == 0) { sm_m[warp] = m; sm_l[warp] = l; }
        }
        __syncthreads();                      // every warp has read its share of the ring
        if (warp == 0 && g == 0) {
            float mx = NEG_BIG;
#pragma unroll
            for (int w = 0; w < SWA_WARPS; ++w) mx = fmaxf(mx, sm_m[w]);
            float L = 0.f, out[EPL];
#pragma unroll
            for (int i = 0; i < EPL; ++i) out[i] = 0.f;
#pragma unroll
            for (int w = 0; w < SWA_WARPS; ++w) {
                float c = exp2f(sm_m[w] - mx);
                L += sm_l[w] * c;
#pragma unroll
                for (int i = 0; i < EPL; ++i) out[i] += sm_acc[w][li * EPL + i] * c;
            }
            if (n_splits == 1) {
                float inv = 1.0f / L;
#pragma unroll
                for (int i = 0; i < EPL; ++i) out[i] *= inv;
                st16(o + (long long)b * d + h * HD + li * EPL, Vec16<T>::pack(out));
            } else {
                float* pp = part + (long long)wi * (HD + 2);
#pragma unroll
                for (int i = 0; i < EPL; ++i) pp[li * EPL + i] = out[i];
                if (li == 0) { pp[HD] = mx; pp[HD + 1] = L; }
            }
            if (W > 1 && writer) {
                st16(Kr + (long long)slot * HD + li * EPL, sm_kv[0][li]);
                st16(Vr + (long long)slot * HD + li * EPL, sm_kv[1][li]);
            }
        }
        __syncthreads();                      // shared partials are free for the next item
    }
}

template <typename T, int HD>
__global__ void __launch_bounds__(WARPS * 32) k_xattn_decode(const float* __restrict__ qc,
                                                             const T* __restrict__ Mg, long long plane,
                                                             int T_alloc, int t, const int32_t* __restrict__ pos,
                                                             T* __restrict__ o, int B, int H,
                                                             int n_splits, int chunk, float* __restrict__ part,
                                                             float qscale) {
    using G = Geom<T, HD>;
    constexpr int EPL = G::EPL, LPK = G::LPK;
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31, g = lane / LPK, li = lane % LPK;
    const int n_items = B * H * n_splits;
    // one (sequence, head, key chunk) item per warp and iteration; a capped grid strides over
    // the items
    for (int item = blockIdx.x * WARPS + (threadIdx.x >> 5); item < n_items; item += gridDim.x * WARPS) {
        int bh = item / n_splits, sp = item % n_splits;
        int b = bh / H, h = bh % H;
        const int d = H * HD;
        float q[EPL];
        const float* qr = qc + (long long)b * d + h * HD + li * EPL;
#pragma unroll
        for (int i = 0; i < EPL; ++i) q[i] = qr[i] * qscale;
        const T* K = Mg + (long long)bh * T_alloc * HD;
        const T* V = K + plane;
        // keys 0 .. tb-1: tb = t for every sequence, or pos[b] + 1 (at most t) per sequence
        const int tb = pos ? min(max(pos[b] + 1, 1), t) : t;
        int j0 = sp * chunk;
        int n = max(0, min(tb, j0 + chunk) - j0);
        float m = NEG_BIG, l = 0.f, acc[EPL];
#pragma unroll
        for (int i = 0; i < EPL; ++i) acc[i] = 0.f;
        attend<T, HD, 4, true>(q, K + (long long)j0 * HD, V + (long long)j0 * HD, n, g, li, m, l, acc);
        merge_groups<T, HD>(m, l, acc);
        if (g != 0) continue;
        if (n_splits == 1) {
            float inv = 1.0f / l, out[EPL];
#pragma unroll
            for (int i = 0; i < EPL; ++i) out[i] = acc[i] * inv;
            st16(o + (long long)b * d + h * HD + li * EPL, Vec16<T>::pack(out));
        } else {
            float* pp = part + (long long)item * (HD + 2);
#pragma unroll
            for (int i = 0; i < EPL; ++i) pp[li * EPL + i] = acc[i];
            if (li == 0) { pp[HD] = m; pp[HD + 1] = l; }
        }
    }
}

// Combine key-split partials: one block per (b, h), one thread per output element.
template <typename T>
__global__ void k_attn_combine(const float* __restrict__ part, int n_splits, int HD, int H,
                               T* __restrict__ o) {
    pdl_wait();
    pdl_trigger();
    int bh = blockIdx.x, c = threadIdx.x;
    if (c >= HD) return;
    const float* p = part + (long long)bh * n_splits * (HD + 2);
    float mx = NEG_BIG;
    for (int s = 0; s < n_splits; ++s) mx = fmaxf(mx, p[s * (HD + 2) + HD]);
    float L = 0.f, A = 0.f;
    for (int s = 0; s < n_splits; ++s) {
        float w = exp2f(p[s * (HD + 2) + HD] - mx);
        L += p[s * (HD + 2) + HD + 1] * w;
        A += p[s * (HD + 2) + c] * w;
    }
    int b = bh / H, h = bh % H;
    o[(long long)b * H * HD + h * HD + c] = from_f<T>(A / L);
}

template <typename T, int HD>
__global__ void __launch_bounds__(WARPS * 32, 8) k_enc_attn(const T* __restrict__ planes, T* __restrict__ o,
                                                         int B, int Tn, int H, float qscale) {
    using G = Geom<T, HD>;
    constexpr int EPL = G::EPL, LPK = G::LPK;
    pdl_wait();
    pdl_trigger();
    long long item = (long long)blockIdx.x * WARPS + (threadIdx.x >> 5);
    if (item >= (long long)B * H * Tn) return;
    int lane = threadIdx.x & 31, g = lane / LPK, li = lane % LPK;
    long long bh = item / Tn;
    int i = (int)(item % Tn);
    long long plane = (long long)B * H * Tn * HD;
    const T* Q = planes + bh * Tn * HD;
    const T* K = planes + plane + bh * Tn * HD;
    const T* V = planes + 2 * plane + bh * Tn * HD;
    float q[EPL];
    Vec16<T>::unpack(ld16(Q + (long long)i * HD + li * EPL), q);
#pragma unroll
    for (int x = 0; x < EPL; ++x) q[x] *= qscale;
    float m = NEG_BIG, l = 0.f, acc[EPL];
#pragma unroll
    for (int x = 0; x < EPL; ++x) acc[x] = 0.f;
    attend<T, HD, 4, false>(q, K, V, i + 1, g, li, m, l, acc);
    merge_groups<T, HD>(m, l, acc);
    if (g != 0) return;
    int b = (int)(bh / H), h = (int)(bh % H);
    float inv = 1.0f / l, out[EPL];
#pragma unroll
    for (int x = 0; x < EPL; ++x) out[x] = acc[x] * inv;
    st16(o + ((long long)b * Tn + i) * H * HD + h * HD + li * EPL, Vec16<T>::pack(out));
}

inline float qscale_for(int hd) { return LOG2E / sqrtf((float)hd); }
inline unsigned blocks_for(long long items) { return (unsigned)((items + WARPS - 1) / WARPS); }
// A grid of `blocks` CTAs, capped at L.attn_ctas_per_sm resident CTAs on every SM when set.
inline unsigned capped(const Launch& L, unsigned blocks) {
    if (L.attn_ctas_per_sm <= 0) return blocks;
    const long long cap = (long long)sm_count() * L.attn_ctas_per_sm;
    return blocks > cap ? (unsigned)cap : blocks;
}

}  // namespace

#define RLT_HD_DISPATCH(hd, EXPR)                                  \
    switch (hd) {                                                  \
        case 16: { constexpr int HD = 16; return EXPR; }           \
        case 32: { constexpr int HD = 32; return EXPR; }           \
        case 64: { constexpr int HD = 64; return EXPR; }           \
        case 128: { constexpr int HD = 128; return EXPR; }         \
        default: return cudaErrorInvalidValue;                     \
    }

template <typename T>
static cudaError_t swa_main(Launch L, const float* qkv, const float2* rope, T* ring, T* o, int B, int H, int hd,
                           int W, const int32_t* pos, int max_t, int n_splits, float* part) {
    RLT_HD_DISPATCH(hd, launch_k(L, k_swa_decode<T, HD>, capped(L, (unsigned)(B * H * n_splits)), SWA_WARPS * 32, 0,
                                 qkv, rope, ring, o, B, H, W, pos, max_t, n_splits, part, qscale_for(hd)));
}

template <typename T>
cudaError_t launch_swa_decode(Launch L, const float* qkv, const float2* rope, T* ring, T* o, int B,
                              int H, int hd, int W, const int32_t* pos, int max_t, int n_splits, float* part) {
    if (n_splits < 1 || !part) n_splits = 1;
    cudaError_t e = swa_main<T>(L, qkv, rope, ring, o, B, H, hd, W, pos, max_t, n_splits, part);
    if (e != cudaSuccess || n_splits == 1) return e;
    return launch_k(L, k_attn_combine<T>, (unsigned)(B * H), (unsigned)hd, 0, (const float*)part, n_splits, hd, H, o);
}

template <typename T>
static cudaError_t xattn_main(Launch L, const float* qc, const T* Mg, long long plane, int T_alloc, int t,
                              const int32_t* pos, T* o, int B, int H, int hd, int n_splits, int chunk, float* part) {
    RLT_HD_DISPATCH(hd, launch_k(L, k_xattn_decode<T, HD>, capped(L, blocks_for((long long)B * H * n_splits)), WARPS * 32, 0,
                                 qc, Mg, plane, T_alloc, t, pos, o, B, H, n_splits, chunk, part, qscale_for(hd)));
}

template <typename T>
cudaError_t launch_xattn_decode(Launch L, const float* qc, const T* Mg, long long plane, int T_alloc, int t, T* o,
                                int B, int H, int hd, int n_splits, float* part, const int32_t* pos) {
    if (n_splits < 1) n_splits = 1;
    int chunk = (t + n_splits - 1) / n_splits;
    cudaError_t e = xattn_main<T>(L, qc, Mg, plane, T_alloc, t, pos, o, B, H, hd, n_splits, chunk, part);
    if (e != cudaSuccess || n_splits == 1) return e;
    return launch_k(L, k_attn_combine<T>, (unsigned)(B * H), (unsigned)hd, 0, (const float*)part, n_splits, hd, H, o);
}

template <typename T>
cudaError_t launch_enc_attention(Launch L, const T* planes, T* o, int B, int Tn, int H, int hd) {
    RLT_HD_DISPATCH(hd, launch_k(L, k_enc_attn<T, HD>, blocks_for((long long)B * H * Tn), WARPS * 32, 0, planes, o,
                                 B, Tn, H, qscale_for(hd)));
}

#define RLT_INST(T)                                                                                    \
    template cudaError_t launch_swa_decode<T>(Launch, const float*, const float2*, T*, T*, int, int,   \
                                              int, int, const int32_t*, int, int, float*);             \
    template cudaError_t launch_xattn_decode<T>(Launch, const float*, const T*, long long, int, int, T*, int, \
                                                int, int, int, float*, const int32_t*);                \
    template cudaError_t launch_enc_attention<T>(Launch, const T*, T*, int, int, int, int);
RLT_INST(float)
RLT_INST(bf16)
#undef RLT_INST

}  // namespace rlt
