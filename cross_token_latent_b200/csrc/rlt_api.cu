// C ABI of the RLT library (declared in include/rlt.h): model arena layout, weight
// packing, the decoder-state registry and the encode / decode-step / replay drivers.
#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <type_traits>
#include <string>
#include <unordered_map>
#include <unordered_set>
#include <vector>

#include "rlt.h"
#include "kernels.cuh"

using namespace rlt;

namespace {

constexpr size_t ALIGN = 256;
inline size_t align_up(size_t x) { return (x + ALIGN - 1) / ALIGN * ALIGN; }
inline bool aligned(const void* p, size_t a = ALIGN) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Batches of at least this many sequences may run a step as two row groups on two streams
// (each group then still fills whole 128-row GEMM tiles).
constexpr int GROUP_MIN_ROWS = 256;

// Cross-attention key-split partials: capacity in (sequence, head, split) work items.
constexpr long long XATTN_PART_ITEMS = 32768;
constexpr int XATTN_MAX_SPLITS = 64;
constexpr int XATTN_MIN_CHUNK = 64;
constexpr long long XATTN_TARGET_WARPS = 148LL * 64 * 2;

struct Layout {
    size_t esz = 0;             // bytes per stored element
    size_t rope = 0, embed = 0, enc_norm = 0, mem = 0, merge_w = 0, merge_b = 0, s_star = 0,
           dec_norm = 0, unembed = 0, total = 0;
    std::vector<size_t> attn_norm, wqkv, wo, ffn_norm, wgu, wdown, xattn_norm, wqc, woc;
};

bool config_ok(const rlt_config& c) {
    if (c.V < 8 || c.d < 8 || c.n_heads < 1 || c.L_E < 1 || c.L_D < 1 || c.F < 8 || c.W < 1) return false;
    if (c.head_dim != 16 && c.head_dim != 32 && c.head_dim != 64 && c.head_dim != 128) return false;
    if (c.n_heads * c.head_dim != c.d) return false;
    if (c.d % 8 || c.F % 8 || c.V % 8) return false;
    if (c.L_E != c.L_D) return false;
    if (c.G != 1 && c.G != c.L_D) return false;
    if (c.dtype != RLT_F32 && c.dtype != RLT_BF16) return false;
    if (c.max_pos < 1 || !(c.rms_eps >= 0.f) || !(c.rope_base > 1.f)) return false;
    return true;
}

Layout make_layout(const rlt_config& c) {
    Layout L;
    L.esz = c.dtype == RLT_BF16 ? 2 : 4;
    size_t off = ALIGN;   // DevHeader
    auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes); return o; };
    size_t d = c.d, F = c.F, V = c.V, e = L.esz;
    L.rope = take((size_t)c.max_pos * (c.head_dim / 2) * sizeof(float2));
    L.embed = take(V * d * e);
    for (int l = 0; l < c.L_E; ++l) {
        L.attn_norm.push_back(take(d * 4));
        L.wqkv.push_back(take(3 * d * d * e));
        L.wo.push_back(take(d * d * e));
        L.ffn_norm.push_back(take(d * 4));
        L.wgu.push_back(take(2 * F * d * e));
        L.wdown.push_back(take(d * F * e));
    }
    L.enc_norm = take(d * 4);
    L.mem = take((size_t)c.G * 2 * d * d * e);
    for (int l = 0; l < c.L_D; ++l) {
        L.xattn_norm.push_back(take(d * 4));
        L.wqc.push_back(take(d * d * e));
        L.woc.push_back(take(d * d * e));
    }
    L.merge_w = take(4 * d * d * e);
    L.merge_b = take(d * 4);
    L.s_star = take(d * 4);
    L.dec_norm = take(d * 4);
    L.unembed = take(V * d * e);
    L.total = off;
    return L;
}

// Host mirror of a registered state: the batch, the model version it was built under and the
// position (tokens consumed) of every row.  The device copy of the positions lives in the state
// buffer and is advanced by the step's kernels in the same way.
struct StateInfo {
    int B = 0;
    uint64_t version = 0;
    std::vector<int64_t> pos;
    int64_t t_max() const {
        int64_t t = 0;
        for (int64_t p : pos) t = p > t ? p : t;
        return t;
    }
    static StateInfo uniform(int B, int64_t t, uint64_t version) {
        StateInfo s;
        s.B = B;
        s.version = version;
        s.pos.assign((size_t)B, t);
        return s;
    }
};

// How one canonical weight maps into the arena.
struct Dest {
    bool ok = false;
    bool vec = false;          // float32 vector copy
    size_t off = 0;            // arena byte offset
    size_t numel = 0;
    int rows = 0, cols = 0, dst_ld = 0, row_mult = 1, row_off = 0, col_off = 0;
    int groups = 1;            // mem_k / mem_v: G separate [d, d] blocks
    size_t group_stride = 0;   // bytes between group blocks in the arena
};

bool parse_layer(const std::string& name, const char* prefix, int& l, std::string& field) {
    size_t n = strlen(prefix);
    if (name.compare(0, n, prefix) != 0) return false;
    size_t dot = name.find('.', n);
    if (dot == std::string::npos || dot == n) return false;
    for (size_t i = n; i < dot; ++i)
        if (name[i] < '0' || name[i] > '9') return false;
    l = std::stoi(name.substr(n, dot - n));
    field = name.substr(dot + 1);
    return true;
}

}  // namespace

// Event pairs around selected launches (rlt_profile_start / rlt_profile_stop).
struct Profiler {
    bool on = false;
    uint32_t mask = 0;
    std::vector<cudaEvent_t> pool;
    size_t used = 0;
    std::vector<std::pair<int, size_t>> recs;   // (kind, index of the start event)

    int begin(int kind, cudaStream_t st) {
        if (!on || !(mask & (1u << kind))) return -1;
        while (pool.size() < used + 2) {
            cudaEvent_t e;
            if (cudaEventCreate(&e) != cudaSuccess) return -1;
            pool.push_back(e);
        }
        size_t i = used;
        used += 2;
        cudaEventRecord(pool[i], st);
        recs.push_back({kind, i});
        return (int)i;
    }
    void end(int i, cudaStream_t st) {
        if (i >= 0) cudaEventRecord(pool[i + 1], st);
    }
    ~Profiler() {
        for (auto e : pool) cudaEventDestroy(e);
    }
};

struct rlt_model {
    Profiler prof;
    rlt_config cfg;
    Layout lay;
    uint8_t* arena = nullptr;
    uint64_t version = 0;
    std::unordered_set<std::string> loaded;
    std::vector<std::string> required;
    std::unordered_map<const void*, StateInfo> states;
    uint64_t launches = 0;
    int device = -1;            // the CUDA device that holds the arena
    // rlt_set_option values
    int opt_row_groups = 1;             // 1 one group, 2 two groups when B >= GROUP_MIN_ROWS
    int opt_attn_cap = 0;               // resident attention CTAs per SM (0: no cap)
    int opt_group_pdl = 0;              // programmatic dependent launch inside a group's chain
    int opt_gemv_rows = 0;              // projections of at most this many rows stream on CUDA cores
    int opt_persistent = 1;             // grids of several waves of 128 x 256 tiles run persistently
    int opt_small_step = 1;             // small models: the whole step in one launch
    // two row groups: library-owned streams, forked from and joined back to the caller's stream
    cudaStream_t gs[2] = {nullptr, nullptr};
    cudaEvent_t fork_ev = nullptr, join_ev[2] = {nullptr, nullptr};

    ~rlt_model() {
        for (int i = 0; i < 2; ++i) {
            if (gs[i]) cudaStreamDestroy(gs[i]);
            if (join_ev[i]) cudaEventDestroy(join_ev[i]);
        }
        if (fork_ev) cudaEventDestroy(fork_ev);
    }
    bool group_streams() {
        if (gs[0]) return true;
        for (int i = 0; i < 2; ++i) {
            if (cudaStreamCreateWithFlags(&gs[i], cudaStreamNonBlocking) != cudaSuccess) return false;
            if (cudaEventCreateWithFlags(&join_ev[i], cudaEventDisableTiming) != cudaSuccess) return false;
        }
        return cudaEventCreateWithFlags(&fork_ev, cudaEventDisableTiming) == cudaSuccess;
    }
    int row_groups(int B) const {
        if (opt_row_groups != 2 || B < GROUP_MIN_ROWS || cfg.dtype != RLT_BF16) return 1;
        return 2;
    }

    DevHeader* hdr() const { return reinterpret_cast<DevHeader*>(arena); }
    template <typename T> T* at(size_t off) const { return reinterpret_cast<T*>(arena + off); }
    Launch launch(void* stream) {
        Launch L{reinterpret_cast<cudaStream_t>(stream), &launches};
        L.gemv_max_rows = opt_gemv_rows;
        L.persistent = opt_persistent != 0;
        return L;
    }

    Dest dest(const std::string& name) const {
        const rlt_config& c = cfg;
        Dest D;
        int d = c.d, F = c.F, V = c.V;
        auto mat = [&](size_t off, int rows, int cols, int dst_ld, int mult, int roff, int coff) {
            D.ok = true; D.off = off; D.rows = rows; D.cols = cols; D.dst_ld = dst_ld;
            D.row_mult = mult; D.row_off = roff; D.col_off = coff; D.numel = (size_t)rows * cols;
        };
        auto vec = [&](size_t off) { D.ok = true; D.vec = true; D.off = off; D.numel = d; };
        int l;
        std::string f;
        if (name == "embed") mat(lay.embed, V, d, d, 1, 0, 0);
        else if (name == "unembed") mat(lay.unembed, V, d, d, 1, 0, 0);
        else if (name == "enc_norm") vec(lay.enc_norm);
        else if (name == "dec_norm") vec(lay.dec_norm);
        else if (name == "s_star") vec(lay.s_star);
        else if (name == "merge_bias") vec(lay.merge_b);
        else if (name == "merge_ge") mat(lay.merge_w, d, d, 2 * d, 2, 0, 0);
        else if (name == "merge_gs") mat(lay.merge_w, d, d, 2 * d, 2, 0, d);
        else if (name == "merge_fb") mat(lay.merge_w, d, d, 2 * d, 2, 1, d);
        else if (name == "mem_k" || name == "mem_v") {
            mat(lay.mem, d, d, d, 1, name == "mem_k" ? 0 : d, 0);
            D.groups = c.G;
            D.group_stride = (size_t)2 * d * d * lay.esz;
            D.numel = (size_t)c.G * d * d;
        } else if (parse_layer(name, "layers.", l, f) && l >= 0 && l < c.L_E) {
            if (f == "attn_norm") vec(lay.attn_norm[l]);
            else if (f == "ffn_norm") vec(lay.ffn_norm[l]);
            else if (f == "wq") mat(lay.wqkv[l], d, d, d, 1, 0, 0);
            else if (f == "wk") mat(lay.wqkv[l], d, d, d, 1, d, 0);
            else if (f == "wv") mat(lay.wqkv[l], d, d, d, 1, 2 * d, 0);
            else if (f == "wo") mat(lay.wo[l], d, d, d, 1, 0, 0);
            else if (f == "w_gate") mat(lay.wgu[l], F, d, d, 2, 0, 0);
            else if (f == "w_up") mat(lay.wgu[l], F, d, d, 2, 1, 0);
            else if (f == "w_down") mat(lay.wdown[l], d, F, F, 1, 0, 0);
        } else if (parse_layer(name, "dec.", l, f) && l >= 0 && l < c.L_D) {
            if (f == "xattn_norm") vec(lay.xattn_norm[l]);
            else if (f == "w_qc") mat(lay.wqc[l], d, d, d, 1, 0, 0);
            else if (f == "w_oc") mat(lay.woc[l], d, d, d, 1, 0, 0);
        }
        return D;
    }
};

namespace {

#define CK(x)                                  \
    do {                                       \
        cudaError_t e__ = (x);                 \
        if (e__ != cudaSuccess) return RLT_ECUDA; \
    } while (0)

// CK() with an optional timing bracket of the given kernel kind.
#define CKP(kind, x)                                   \
    do {                                               \
        int p__ = m->prof.begin((kind), L.stream);     \
        cudaError_t e__ = (x);                         \
        m->prof.end(p__, L.stream);                    \
        if (e__ != cudaSuccess) return RLT_ECUDA;      \
    } while (0)

size_t state_s_off() { return ALIGN; }
size_t state_ring_off(const rlt_config& c, int B) { return align_up(ALIGN + (size_t)B * c.d * 4); }
size_t ring_layer_elems(const rlt_config& c, int B) {
    return (size_t)B * 2 * c.n_heads * (size_t)(c.W - 1) * c.head_dim;
}
size_t state_pos_off(const rlt_config& c, int B) {
    return align_up(state_ring_off(c, B) + (size_t)c.L_D * ring_layer_elems(c, B) * (c.dtype == RLT_BF16 ? 2 : 4));
}
int32_t* state_pos(const rlt_config& c, uint8_t* state, int B) {
    return reinterpret_cast<int32_t*>(state + state_pos_off(c, B));
}

struct EncWS {
    size_t h, a, act, qkv, planes, att, ews, total;
};
EncWS enc_ws(const rlt_config& c, int B, int T) {
    EncWS w;
    size_t N = (size_t)B * T, d = c.d, e = c.dtype == RLT_BF16 ? 2 : 4;
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes); return o; };
    w.h = take(N * d * 4);
    w.a = take(N * d * e);
    w.act = take(N * (size_t)c.F * e);
    w.qkv = take(N * 3 * d * 4);
    // q and k planes, then v ([B][H][T][hd]) or, on the tensor-core path, v transposed
    // ([B][H][hd][T_pad])
    w.planes = take(2 * N * d * e + (size_t)B * c.n_heads * c.head_dim * enc_vt_pitch(T) * e);
    w.att = take(N * d * e);
    w.ews = take(N * d * e);
    w.total = off;
    return w;
}

struct DecWS {
    size_t x, A, qkv, att, qc, act, logits, part, part2, xn, ss, total;
};
DecWS dec_ws(const rlt_config& c, int B) {
    DecWS w;
    size_t d = c.d, e = c.dtype == RLT_BF16 ? 2 : 4;
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes); return o; };
    w.x = take((size_t)B * d * 4);
    w.A = take((size_t)B * 2 * d * e);
    w.qkv = take((size_t)B * 3 * d * 4);
    w.att = take((size_t)B * d * e);
    w.qc = take((size_t)B * d * 4);
    w.act = take((size_t)B * c.F * e);
    w.logits = take((size_t)B * c.V * 4);
    w.part = take((size_t)XATTN_PART_ITEMS * (c.head_dim + 2) * 4);
    // the second row group's key-split partials
    w.part2 = B >= GROUP_MIN_ROWS ? take((size_t)XATTN_PART_ITEMS * (c.head_dim + 2) * 4) : w.part;
    w.xn = take((size_t)B * d * e);               // bf16(x * g) of a deferred norm
    w.ss = take((size_t)B * (d / 16) * 4);        // its 16-column sum-of-squares partials
    w.total = off;
    return w;
}

// Key splits of the decoder's sliding-window attention: one CTA per (sequence, head) fills
// the GPU at large batches; below ~6 CTAs per SM the window is cut into ranges of at least 32
// cached entries, one CTA each.
int swa_splits(const rlt_config& c, int B, int t) {
    const long long bh = (long long)B * c.n_heads;
    const int n = std::min(t - 1, c.W - 1);
    const long long want = (148LL * 6 + bh - 1) / bh;
    long long s = std::min<long long>(want, (n + 31) / 32);
    s = std::min<long long>(s, std::min<long long>(16, XATTN_PART_ITEMS / bh));
    return s < 1 ? 1 : (int)s;
}

int xattn_splits(const rlt_config& c, int B, int t) {
    long long bh = (long long)B * c.n_heads;
    // enough (sequence, head) pairs for 32 warps per SM: no split (300M B=512: 8192 pairs,
    // measured faster unsplit than in three chunks, and no combine launch)
    if (bh >= 148LL * 32) return 1;
    long long want = (XATTN_TARGET_WARPS + bh - 1) / bh;
    // few (sequence, head) pairs: shorter chunks, so that more warps stream the keys
    const int min_chunk = bh < 592 ? XATTN_MIN_CHUNK / 2 : XATTN_MIN_CHUNK;
    long long by_len = (t + min_chunk - 1) / min_chunk;
    long long cap = XATTN_PART_ITEMS / bh;
    long long s = want;
    if (s > by_len) s = by_len;
    if (s > XATTN_MAX_SPLITS) s = XATTN_MAX_SPLITS;
    if (s > cap) s = cap;
    return s < 1 ? 1 : (int)s;
}

// ------------------------------------------------------------------ encoder driver
size_t enc_cache_layer_elems(const rlt_config& c, int B, int T_max) {
    return (size_t)2 * B * c.n_heads * (size_t)T_max * c.head_dim;
}

// Token-parallel encoder over Tn tokens of B sequences; with `cache` (capacity T_max) it also
// stores every layer's rotated keys and values of positions 0..Tn-1 for incremental appends.
template <typename T>
rlt_status encode_impl(rlt_model* m, const int32_t* tokens, int B, int Tn, int T_alloc, T* e, T* M,
                       uint8_t* ws, cudaStream_t st, T* cache = nullptr, int T_max = 0) {
    const rlt_config& c = m->cfg;
    Launch L = m->launch(st);
    EncWS w = enc_ws(c, B, Tn);
    int N = B * Tn, d = c.d, F = c.F, H = c.n_heads, hd = c.head_dim;
    float* h = reinterpret_cast<float*>(ws + w.h);
    T* a = reinterpret_cast<T*>(ws + w.a);
    T* act = reinterpret_cast<T*>(ws + w.act);
    float* qkv = reinterpret_cast<float*>(ws + w.qkv);
    T* planes = reinterpret_cast<T*>(ws + w.planes);
    T* att = reinterpret_cast<T*>(ws + w.att);
    T* ews = reinterpret_cast<T*>(ws + w.ews);
    const float2* rope = m->at<float2>(m->lay.rope);
    const bool use_tc_attn = sizeof(T) == 2 && enc_attention_tc_supported(hd);
    CKP(RLT_K_ENC_OTHER, launch_embed<T>(L, tokens, N, m->at<T>(m->lay.embed), c.V, d, h, m->hdr()));
    for (int l = 0; l < c.L_E; ++l) {
        EpiArgs ea; ea.hdr = m->hdr();
        CKP(RLT_K_ENC_OTHER, launch_rmsnorm<T>(L, h, N, d, m->at<float>(m->lay.attn_norm[l]), c.rms_eps, a, d, N, N, nullptr));
        ea.out_f32 = qkv; ea.ld_out = 3 * d;
        CKP(RLT_K_ENC_GEMM, launch_gemm<T>(L, Epi::StoreF32, a, d, m->at<T>(m->lay.wqkv[l]), N, 3 * d, d, ea));
        if (cache)
            CKP(RLT_K_ENC_OTHER, launch_enc_cache_write<T>(L, qkv, B, Tn, H, hd, rope, 0, nullptr,
                                         cache + (size_t)l * enc_cache_layer_elems(c, B, T_max), T_max, nullptr));
        if (use_tc_attn) {
            bf16* pl = reinterpret_cast<bf16*>(planes);
            size_t plane = (size_t)N * d;
            CKP(RLT_K_ENC_OTHER, launch_enc_qkv_layout<T>(L, qkv, B, Tn, H, hd, rope, planes, false));
            CKP(RLT_K_ENC_OTHER, launch_enc_vt(L, qkv, pl + 2 * plane, B, Tn, H, hd));
            CKP(RLT_K_ENC_ATTN, launch_enc_attention_tc(L, pl, pl + plane, pl + 2 * plane, reinterpret_cast<bf16*>(att), B, Tn, H, hd,
                                       m->hdr()));
        } else {
            CKP(RLT_K_ENC_OTHER, launch_enc_qkv_layout<T>(L, qkv, B, Tn, H, hd, rope, planes));
            CKP(RLT_K_ENC_ATTN, launch_enc_attention<T>(L, planes, att, B, Tn, H, hd));
        }
        ea = EpiArgs(); ea.hdr = m->hdr(); ea.out_f32 = h; ea.ld_out = d;
        CKP(RLT_K_ENC_GEMM, launch_gemm<T>(L, Epi::ResidAdd, att, d, m->at<T>(m->lay.wo[l]), N, d, d, ea));
        CKP(RLT_K_ENC_OTHER, launch_rmsnorm<T>(L, h, N, d, m->at<float>(m->lay.ffn_norm[l]), c.rms_eps, a, d, N, N, nullptr));
        ea = EpiArgs(); ea.hdr = m->hdr(); ea.out_t = act; ea.ld_out = F;
        CKP(RLT_K_ENC_GEMM, launch_gemm<T>(L, Epi::SwiGLU, a, d, m->at<T>(m->lay.wgu[l]), N, 2 * F, d, ea));
        ea = EpiArgs(); ea.hdr = m->hdr(); ea.out_f32 = h; ea.ld_out = d;
        CKP(RLT_K_ENC_GEMM, launch_gemm<T>(L, Epi::ResidAdd, act, F, m->at<T>(m->lay.wdown[l]), N, d, F, ea));
    }
    // e = RMSNorm(h) written with row capacity T_alloc, plus a contiguous copy for M
    CKP(RLT_K_ENC_OTHER, launch_rmsnorm<T>(L, h, N, d, m->at<float>(m->lay.enc_norm), c.rms_eps, e, d, Tn, T_alloc, ews));
    size_t group_elems = (size_t)2 * B * H * (size_t)T_alloc * hd;
    for (int g = 0; g < c.G; ++g) {
        EpiArgs ea; ea.hdr = m->hdr();
        ea.out_f32 = qkv; ea.ld_out = 2 * d;
        CKP(RLT_K_ENC_GEMM, launch_gemm<T>(L, Epi::StoreF32, ews, d, m->at<T>(m->lay.mem) + (size_t)g * 2 * d * d, N, 2 * d, d, ea));
        CKP(RLT_K_ENC_OTHER, launch_mem_layout<T>(L, qkv, B, Tn, T_alloc, H, hd, M + g * group_elems));
    }
    return RLT_OK;
}

// ------------------------------------------------------------------ incremental encoder
struct AppWS {
    size_t h, a, act, qkv, q, att, ews, part, total;
};
AppWS app_ws(const rlt_config& c, int B) {
    AppWS w;
    size_t d = c.d, e = c.dtype == RLT_BF16 ? 2 : 4;
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes); return o; };
    w.h = take((size_t)B * d * 4);
    w.a = take((size_t)B * d * e);
    w.act = take((size_t)B * c.F * e);
    w.qkv = take((size_t)B * 3 * d * 4);
    w.q = take((size_t)B * d * 4);
    w.att = take((size_t)B * d * e);
    w.ews = take((size_t)B * d * e);
    w.part = take((size_t)XATTN_PART_ITEMS * (c.head_dim + 2) * 4);
    w.total = off;
    return w;
}

// One new token per sequence at position pos: the encoder layers run on B rows, each layer's
// causal attention reads the cached keys/values of positions 0..pos (the new ones written
// first), and the new encoder output and memory rows go to e[:, pos] and M[..., pos, :].
template <typename T>
rlt_status encode_append_impl(rlt_model* m, const int32_t* tok, int tok_stride, int B, int pos,
                              const int32_t* positions, T* cache, int T_max, T* e, T* M, int T_alloc, uint8_t* ws,
                              cudaStream_t st) {
    const rlt_config& c = m->cfg;
    Launch L = m->launch(st);
    AppWS w = app_ws(c, B);
    const int d = c.d, F = c.F, H = c.n_heads, hd = c.head_dim;
    float* h = reinterpret_cast<float*>(ws + w.h);
    T* a = reinterpret_cast<T*>(ws + w.a);
    T* act = reinterpret_cast<T*>(ws + w.act);
    float* qkv = reinterpret_cast<float*>(ws + w.qkv);
    float* q = reinterpret_cast<float*>(ws + w.q);
    T* att = reinterpret_cast<T*>(ws + w.att);
    T* ews = reinterpret_cast<T*>(ws + w.ews);
    float* part = reinterpret_cast<float*>(ws + w.part);
    const float2* rope = m->at<float2>(m->lay.rope);
    const long long cplane = (long long)B * H * T_max * hd;
    const int splits = xattn_splits(c, B, pos + 1);
    int p = m->prof.begin(RLT_K_ENCODER, st);
    CK(launch_embed<T>(L, tok, B, m->at<T>(m->lay.embed), c.V, d, h, m->hdr(), tok_stride));
    for (int l = 0; l < c.L_E; ++l) {
        T* cache_l = cache + (size_t)l * enc_cache_layer_elems(c, B, T_max);
        EpiArgs ea; ea.hdr = m->hdr();
        CK(launch_rmsnorm<T>(L, h, B, d, m->at<float>(m->lay.attn_norm[l]), c.rms_eps, a, d, B, B, nullptr));
        ea.out_f32 = qkv; ea.ld_out = 3 * d;
        CK(launch_gemm<T>(L, Epi::StoreF32, a, d, m->at<T>(m->lay.wqkv[l]), B, 3 * d, d, ea));
        CK(launch_enc_cache_write<T>(L, qkv, B, 1, H, hd, rope, pos, positions, cache_l, T_max, q));
        CK(launch_xattn_decode<T>(L, q, cache_l, cplane, T_max, pos + 1, att, B, H, hd, splits, part, positions));
        ea = EpiArgs(); ea.hdr = m->hdr(); ea.out_f32 = h; ea.ld_out = d;
        CK(launch_gemm<T>(L, Epi::ResidAdd, att, d, m->at<T>(m->lay.wo[l]), B, d, d, ea));
        CK(launch_rmsnorm<T>(L, h, B, d, m->at<float>(m->lay.ffn_norm[l]), c.rms_eps, a, d, B, B, nullptr));
        ea = EpiArgs(); ea.hdr = m->hdr(); ea.out_t = act; ea.ld_out = F;
        CK(launch_gemm<T>(L, Epi::SwiGLU, a, d, m->at<T>(m->lay.wgu[l]), B, 2 * F, d, ea));
        ea = EpiArgs(); ea.hdr = m->hdr(); ea.out_f32 = h; ea.ld_out = d;
        CK(launch_gemm<T>(L, Epi::ResidAdd, act, F, m->at<T>(m->lay.wdown[l]), B, d, F, ea));
    }
    // e[:, pos] = RMSNorm(h) (row b lands at b * T_alloc + pos, or + positions[b]), plus a
    // contiguous copy for M
    if (positions)
        CK(launch_rmsnorm<T>(L, h, B, d, m->at<float>(m->lay.enc_norm), c.rms_eps, e, d, 1, T_alloc, ews, positions));
    else
        CK(launch_rmsnorm<T>(L, h, B, d, m->at<float>(m->lay.enc_norm), c.rms_eps, e + (size_t)pos * d, d, 1, T_alloc,
                             ews));
    const size_t group_elems = (size_t)2 * B * H * (size_t)T_alloc * hd;
    for (int g = 0; g < c.G; ++g) {
        EpiArgs ea; ea.hdr = m->hdr();
        ea.out_f32 = qkv; ea.ld_out = 2 * d;
        CK(launch_gemm<T>(L, Epi::StoreF32, ews, d, m->at<T>(m->lay.mem) + (size_t)g * 2 * d * d, B, 2 * d, d, ea));
        if (positions)
            CK(launch_mem_layout<T>(L, qkv, B, 1, T_alloc, H, hd, M + g * group_elems, positions));
        else
            CK(launch_mem_layout<T>(L, qkv, B, 1, T_alloc, H, hd, M + g * group_elems + (size_t)pos * hd));
    }
    m->prof.end(p, st);
    return RLT_OK;
}

// ------------------------------------------------------------------ one decoder step
struct StepIO {
    const int32_t* tok = nullptr;
    int tok_stride = 1;
    float* logp_tok = nullptr;
    int lp_stride = 1;
    float* lse = nullptr;
    float* logp_full = nullptr;
    float* score = nullptr;
    const int32_t* prompt_len = nullptr;
    float tau = 1.f;
    bool head = true;
};

// Rows [b0, b0 + Bg) of a step over a batch of B sequences: every row-indexed buffer is offset
// by b0; `part` is this row group's key-split buffer; `first` says whether this group checks
// and advances the state header.  Sequence b takes its own step pos[b] + 1 (the positions
// live in the state); t is the largest of those steps (it sizes the key splits and bounds
// every position).
template <typename T>
rlt_status step_rows(rlt_model* m, uint8_t* state, int B, int b0, int Bg, const T* e, const T* M, int T_alloc,
                     int t, const StepIO& io, uint8_t* ws, float* part, bool first, Launch L) {
    const rlt_config& c = m->cfg;
    DecWS w = dec_ws(c, B);
    int d = c.d, F = c.F, H = c.n_heads, hd = c.head_dim;
    const size_t rb = (size_t)b0;
    StateHeader* sh = first ? reinterpret_cast<StateHeader*>(state) : nullptr;
    float* s = reinterpret_cast<float*>(state + state_s_off()) + rb * d;
    T* ring = reinterpret_cast<T*>(state + state_ring_off(c, B)) + rb * 2 * H * (size_t)(c.W - 1) * hd;
    int32_t* pos = state_pos(c, state, B) + rb;
    float* x = reinterpret_cast<float*>(ws + w.x) + rb * d;
    T* A = reinterpret_cast<T*>(ws + w.A) + rb * 2 * d;
    float* qkv = reinterpret_cast<float*>(ws + w.qkv) + rb * 3 * d;
    T* att = reinterpret_cast<T*>(ws + w.att) + rb * d;
    float* qc = reinterpret_cast<float*>(ws + w.qc) + rb * d;
    T* act = reinterpret_cast<T*>(ws + w.act) + rb * F;
    float* logits = reinterpret_cast<float*>(ws + w.logits) + rb * c.V;
    const float2* rope = m->at<float2>(m->lay.rope);
    const size_t group_elems = (size_t)2 * B * H * (size_t)T_alloc * hd;
    const long long plane = (long long)B * H * T_alloc * hd;        // keys -> values of one memory group
    const T* eg = e + rb * T_alloc * d;
    const T* Mrows = M + rb * H * (size_t)T_alloc * hd;
    int splits = xattn_splits(c, Bg, t);

    // Deferred RMSNorm (bf16 tensor-core path): the GEMM that updates the residual stream x
    // also writes bf16(x * g) and per-row sum-of-squares partials, and the GEMM that consumes
    // the norm scales its accumulator rows by 1 / rms (row scaling commutes with the product),
    // so the three sublayer norms of a layer need no launches of their own.
    T* xn = reinterpret_cast<T*>(ws + w.xn) + rb * d;
    float* ss = reinterpret_cast<float*>(ws + w.ss) + rb * (d / 16);
    const bool fuse = std::is_same<T, bf16>::value && d % 64 == 0 &&
                      gemm_tc_supported(xn, d, m->at<T>(m->lay.wqkv[0]), d) &&
                      gemm_tc_supported(A, 2 * d, m->at<T>(m->lay.merge_w), 2 * d) &&
                      gemm_tc_supported(att, d, m->at<T>(m->lay.wo[0]), d) &&
                      gemm_tc_supported(act, F, m->at<T>(m->lay.wdown[0]), F);
    auto norm_out = [&](EpiArgs& ea, const float* g) {
        if (!fuse) return;
        ea.norm_y = reinterpret_cast<bf16*>(xn); ea.norm_g = g; ea.ss_out = ss; ea.ss_ld = d / 16;
    };
    auto norm_in = [&](EpiArgs& ea) {
        if (!fuse) return;
        ea.ss_in = ss; ea.ss_ld = d / 16; ea.ss_n = d / 16; ea.norm_n = (float)d; ea.eps = c.rms_eps;
    };
    // the sublayer input: bf16(x * g) under a deferred norm, else RMSNorm(x) * g from its own kernel
    auto pre_norm = [&](const float* g) -> cudaError_t {
        return launch_rmsnorm<T>(L, x, Bg, d, g, c.rms_eps, A, d, Bg, Bg, nullptr);
    };
    const T* hin = fuse ? xn : A;

    // gated merge: x = e_t + sigmoid(W_ge e_t + W_gs s + b_g) * (W_fb s)
    CKP(RLT_K_MERGE, launch_merge_prep<T>(L, eg, T_alloc, pos, s, A, Bg, d, sh, m->version, m->hdr()));
    {
        EpiArgs ea; ea.hdr = m->hdr();
        ea.out_f32 = x; ea.ld_out = d; ea.merge_e = A; ea.ld_e = 2 * d; ea.bias = m->at<float>(m->lay.merge_b);
        norm_out(ea, m->at<float>(m->lay.attn_norm[0]));
        CKP(RLT_K_MERGE, launch_gemm<T>(L, Epi::Merge, A, 2 * d, m->at<T>(m->lay.merge_w), Bg, 2 * d, 2 * d, ea));
    }
    for (int l = 0; l < c.L_D; ++l) {
        EpiArgs ea; ea.hdr = m->hdr();
        // sliding-window self-attention (weights of encoder layer l)
        if (!fuse) CKP(RLT_K_NORM, pre_norm(m->at<float>(m->lay.attn_norm[l])));
        ea.out_f32 = qkv; ea.ld_out = 3 * d;
        norm_in(ea);
        CKP(RLT_K_QKV, launch_gemm<T>(L, Epi::StoreF32, hin, d, m->at<T>(m->lay.wqkv[l]), Bg, 3 * d, d, ea));
        CKP(RLT_K_SWA, launch_swa_decode<T>(L, qkv, rope, ring + (size_t)l * ring_layer_elems(c, B), att, Bg, H,
                                            hd, c.W, pos, t, swa_splits(c, Bg, t), part));
        ea = EpiArgs(); ea.hdr = m->hdr(); ea.out_f32 = x; ea.ld_out = d;
        norm_out(ea, m->at<float>(m->lay.xattn_norm[l]));
        CKP(RLT_K_O, launch_gemm<T>(L, Epi::ResidAdd, att, d, m->at<T>(m->lay.wo[l]), Bg, d, d, ea));
        // cross-attention to M_{<=t}
        if (!fuse) CKP(RLT_K_NORM, pre_norm(m->at<float>(m->lay.xattn_norm[l])));
        ea = EpiArgs(); ea.hdr = m->hdr(); ea.out_f32 = qc; ea.ld_out = d;
        norm_in(ea);
        CKP(RLT_K_QC, launch_gemm<T>(L, Epi::StoreF32, hin, d, m->at<T>(m->lay.wqc[l]), Bg, d, d, ea));
        const T* Mg = Mrows + (c.G == 1 ? 0 : (size_t)l * group_elems);
        CKP(RLT_K_XATTN, launch_xattn_decode<T>(L, qc, Mg, plane, T_alloc, t, att, Bg, H, hd, splits, part, pos));
        ea = EpiArgs(); ea.hdr = m->hdr(); ea.out_f32 = x; ea.ld_out = d;
        norm_out(ea, m->at<float>(m->lay.ffn_norm[l]));
        CKP(RLT_K_OC, launch_gemm<T>(L, Epi::ResidAdd, att, d, m->at<T>(m->lay.woc[l]), Bg, d, d, ea));
        // SwiGLU FFN (weights of encoder layer l)
        if (!fuse) CKP(RLT_K_NORM, pre_norm(m->at<float>(m->lay.ffn_norm[l])));
        ea = EpiArgs(); ea.hdr = m->hdr(); ea.out_t = act; ea.ld_out = F;
        norm_in(ea);
        CKP(RLT_K_FFN_UP, launch_gemm<T>(L, Epi::SwiGLU, hin, d, m->at<T>(m->lay.wgu[l]), Bg, 2 * F, d, ea));
        ea = EpiArgs(); ea.hdr = m->hdr(); ea.out_f32 = x; ea.ld_out = d;
        if (l + 1 < c.L_D) norm_out(ea, m->at<float>(m->lay.attn_norm[l + 1]));
        CKP(RLT_K_FFN_DOWN, launch_gemm<T>(L, Epi::ResidAdd, act, F, m->at<T>(m->lay.wdown[l]), Bg, d, F, ea));
    }
    // split: s_t = RMSNorm(x) becomes the state; the same s_t feeds the head
    CKP(RLT_K_FINAL, launch_final_norm<T>(L, x, Bg, d, m->at<float>(m->lay.dec_norm), c.rms_eps, s, A, sh, t, pos));
    const int32_t* tok = io.tok ? io.tok + rb * io.tok_stride : nullptr;
    float* lp_tok = io.logp_tok ? io.logp_tok + rb * io.lp_stride : nullptr;
    float* lse = io.lse ? io.lse + rb : nullptr;
    float* score = io.score ? io.score + rb : nullptr;
    const int32_t* plen = io.prompt_len ? io.prompt_len + rb : nullptr;
    if (io.head && fuse && Bg > 64 && !io.logp_full) {
        // the head GEMM's epilogue reduces each row tile of logits to (max, sum of exp) partials
        // and the gathered target logit; a small kernel merges them into LSE and log-probs
        EpiArgs ea; ea.hdr = m->hdr();
        ea.scale = 1.0f / io.tau;
        ea.lse_tok = tok; ea.tok_stride = io.tok_stride;
        ea.lse_part = reinterpret_cast<float2*>(logits);
        ea.z_tok = logits + (size_t)Bg * c.V - Bg;      // the last Bg floats of this group's rows
        int n_tiles = 0;
        CKP(RLT_K_HEAD, launch_gemm_tc_lse(L, reinterpret_cast<const bf16*>(A), d,
                                           reinterpret_cast<const bf16*>(m->at<T>(m->lay.unembed)), Bg, c.V, d, ea,
                                           m->hdr(), &n_tiles));
        CKP(RLT_K_LSE, launch_lse_combine(L, ea.lse_part, n_tiles, ea.z_tok, Bg, c.V, tok, io.tok_stride, lp_tok,
                                          io.lp_stride, lse, score, plen, pos, m->hdr()));
    } else if (io.head) {
        EpiArgs ea; ea.hdr = m->hdr();
        ea.out_f32 = logits; ea.ld_out = c.V;
        CKP(RLT_K_HEAD, launch_gemm<T>(L, Epi::StoreF32, A, d, m->at<T>(m->lay.unembed), Bg, c.V, d, ea));
        CKP(RLT_K_LSE, launch_lse_gather(L, logits, Bg, c.V, io.tau, tok, io.tok_stride, lp_tok, io.lp_stride, lse,
                                         io.logp_full ? io.logp_full + rb * c.V : nullptr, score, plen, pos,
                                         m->hdr()));
    }
    return RLT_OK;
}

// One decoder step of all B sequences.  Large batches run as two row groups, each on a
// library stream forked from `st` (an event) and joined back into it: while one group's
// attention streams HBM, the other group's projections run on the tensor cores.  The
// attention grids of both groups are capped so that every SM keeps room for the other
// group's GEMM CTAs.
// A small model's whole step in one launch (small_step.cu): one CTA per sequence.
template <typename T>
rlt_status small_step(rlt_model* m, uint8_t* state, int B, const T* e, const T* M, int T_alloc, int t,
                      const StepIO& io, cudaStream_t st) {
    const rlt_config& c = m->cfg;
    const Layout& y = m->lay;
    SmallStepArgs a = {};
    a.B = B; a.d = c.d; a.H = c.n_heads; a.F = c.F; a.V = c.V; a.W = c.W; a.G = c.G; a.L = c.L_D;
    a.eps = c.rms_eps; a.tau = io.tau;
    a.e = e; a.T_alloc = T_alloc; a.M = M;
    a.plane = (long long)B * c.n_heads * T_alloc * c.head_dim;
    a.group_elems = (size_t)2 * B * c.n_heads * (size_t)T_alloc * c.head_dim;
    a.s = reinterpret_cast<float*>(state + state_s_off());
    a.ring = state + state_ring_off(c, B);
    a.ring_layer = ring_layer_elems(c, B);
    a.pos = state_pos(c, state, B);
    a.sh = reinterpret_cast<StateHeader*>(state);
    a.t_host = t;
    a.version = m->version;
    a.hdr = m->hdr();
    a.rope = m->at<float2>(y.rope);
    a.w.merge = m->at<T>(y.merge_w); a.w.merge_b = m->at<float>(y.merge_b);
    a.w.dec_norm = m->at<float>(y.dec_norm); a.w.unembed = m->at<T>(y.unembed);
    for (int l = 0; l < c.L_D; ++l) {
        a.w.attn_norm[l] = m->at<float>(y.attn_norm[l]);
        a.w.xattn_norm[l] = m->at<float>(y.xattn_norm[l]);
        a.w.ffn_norm[l] = m->at<float>(y.ffn_norm[l]);
        a.w.wqkv[l] = m->at<T>(y.wqkv[l]); a.w.wo[l] = m->at<T>(y.wo[l]);
        a.w.wqc[l] = m->at<T>(y.wqc[l]); a.w.woc[l] = m->at<T>(y.woc[l]);
        a.w.wgu[l] = m->at<T>(y.wgu[l]); a.w.wdown[l] = m->at<T>(y.wdown[l]);
    }
    a.head = io.head;
    a.tok = io.tok; a.tok_stride = io.tok_stride; a.logp_tok = io.logp_tok; a.lp_stride = io.lp_stride;
    a.lse = io.lse; a.logp_full = io.logp_full; a.score = io.score; a.prompt_len = io.prompt_len;
    Launch L = m->launch(st);
    CKP(RLT_K_SMALL_STEP, launch_small_step<T>(L, a, c.head_dim));
    return RLT_OK;
}

template <typename T>
rlt_status step_impl(rlt_model* m, uint8_t* state, int B, const T* e, const T* M, int T_alloc, int t,
                     const StepIO& io, uint8_t* ws, cudaStream_t st) {
    const rlt_config& c = m->cfg;
    if (m->opt_small_step && small_step_supported(c.d, c.F, c.V, c.head_dim, c.L_D))
        return small_step<T>(m, state, B, e, M, T_alloc, t, io, st);
    DecWS w = dec_ws(m->cfg, B);
    float* part = reinterpret_cast<float*>(ws + w.part);
    if (m->row_groups(B) == 1 || !m->group_streams()) {
        Launch L = m->launch(st);
        L.attn_ctas_per_sm = m->opt_attn_cap;
        return step_rows<T>(m, state, B, 0, B, e, M, T_alloc, t, io, ws, part, true, L);
    }
    float* part2 = reinterpret_cast<float*>(ws + w.part2);
    const int B0 = (B / 2 + 127) / 128 * 128;           // group 0: whole 128-row tiles
    CK(cudaEventRecord(m->fork_ev, st));
    rlt_status r = RLT_OK;
    for (int g = 0; g < 2 && r == RLT_OK; ++g) {
        CK(cudaStreamWaitEvent(m->gs[g], m->fork_ev, 0));
        Launch L = m->launch(m->gs[g]);
        L.pdl = m->opt_group_pdl != 0;
        L.attn_ctas_per_sm = m->opt_attn_cap;
        r = g == 0 ? step_rows<T>(m, state, B, 0, B0, e, M, T_alloc, t, io, ws, part, true, L)
                   : step_rows<T>(m, state, B, B0, B - B0, e, M, T_alloc, t, io, ws, part2, false, L);
    }
    // join both groups back into the caller's stream (also after an error: nothing is left
    // dangling on the library streams)
    for (int g = 0; g < 2; ++g) {
        CK(cudaEventRecord(m->join_ev[g], m->gs[g]));
        CK(cudaStreamWaitEvent(st, m->join_ev[g], 0));
    }
    return r;
}

template <typename T>
rlt_status state_init_impl(rlt_model* m, uint8_t* state, int B, cudaStream_t st) {
    Launch L = m->launch(st);
    CK(launch_state_init(L, m->at<float>(m->lay.s_star), B, m->cfg.d,
                         reinterpret_cast<float*>(state + state_s_off()),
                         reinterpret_cast<StateHeader*>(state), m->version, state_pos(m->cfg, state, B)));
    return RLT_OK;
}

size_t replay_e_bytes(const rlt_config& c, int B, int T) {
    return align_up((size_t)B * T * c.d * (c.dtype == RLT_BF16 ? 2 : 4));
}
size_t replay_M_bytes(const rlt_config& c, int B, int T) {
    return align_up((size_t)c.G * 2 * B * (size_t)T * c.d * (c.dtype == RLT_BF16 ? 2 : 4));
}

}  // namespace

// ====================================================================== public API

extern "C" {

const char* rlt_status_string(rlt_status s) {
    switch (s) {
        case RLT_OK: return "ok";
        case RLT_EINVAL: return "invalid argument";
        case RLT_ECUDA: return "CUDA error";
        case RLT_ESTALE: return "state is stale (weights were replaced since it was built)";
        case RLT_ETIMEOUT: return "device wait timed out";
        case RLT_EUNSUPPORTED: return "unsupported shape";
        case RLT_EDEVICE: return "device-side check failed";
        case RLT_ESTATE: return "state not registered with this model or wrong batch";
    }
    return "unknown status";
}

size_t rlt_weights_bytes(const rlt_config* cfg) {
    if (!cfg || !config_ok(*cfg)) return 0;
    return make_layout(*cfg).total;
}

rlt_status rlt_model_create(const rlt_config* cfg, void* arena, size_t arena_bytes, void* stream,
                            rlt_model** out) {
    if (!cfg || !out || !arena || !config_ok(*cfg) || !aligned(arena)) return RLT_EINVAL;
    Layout lay = make_layout(*cfg);
    if (arena_bytes < lay.total) return RLT_EINVAL;
    cudaPointerAttributes pa;
    if (cudaPointerGetAttributes(&pa, arena) != cudaSuccess || pa.type != cudaMemoryTypeDevice) {
        cudaGetLastError();
        return RLT_EINVAL;
    }
    rlt_model* m = new rlt_model();
    m->device = pa.device;
    m->cfg = *cfg;
    m->lay = lay;
    m->arena = reinterpret_cast<uint8_t*>(arena);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(arena, 0, lay.total, st) != cudaSuccess ||
        launch_rope_table(m->launch(stream), m->at<float2>(lay.rope), cfg->max_pos, cfg->head_dim,
                          cfg->rope_base) != cudaSuccess) {
        delete m;
        return RLT_ECUDA;
    }
    const char* fixed[] = {"embed", "enc_norm", "mem_k", "mem_v", "merge_ge", "merge_gs", "merge_fb",
                           "merge_bias", "s_star", "dec_norm", "unembed"};
    for (const char* n : fixed) m->required.push_back(n);
    const char* lf[] = {"attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w_gate", "w_up", "w_down"};
    for (int l = 0; l < cfg->L_E; ++l)
        for (const char* f : lf) m->required.push_back("layers." + std::to_string(l) + "." + f);
    const char* df[] = {"xattn_norm", "w_qc", "w_oc"};
    for (int l = 0; l < cfg->L_D; ++l)
        for (const char* f : df) m->required.push_back("dec." + std::to_string(l) + "." + f);
    *out = m;
    return RLT_OK;
}

void rlt_model_destroy(rlt_model* m) { delete m; }

rlt_status rlt_model_set_weight(rlt_model* m, const char* name, const float* src, size_t numel, void* stream) {
    if (!m || !name || !src || !aligned(src, 16)) return RLT_EINVAL;
    std::string n(name);
    Dest D = m->dest(n);
    if (!D.ok || D.numel != numel) return RLT_EINVAL;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    Launch L = m->launch(stream);
    if (D.vec) {
        CK(cudaMemcpyAsync(m->arena + D.off, src, numel * 4, cudaMemcpyDeviceToDevice, st));
    } else {
        for (int g = 0; g < D.groups; ++g) {
            const float* s = src + (size_t)g * D.rows * D.cols;
            uint8_t* dst = m->arena + D.off + g * D.group_stride;
            cudaError_t e = m->cfg.dtype == RLT_BF16
                ? launch_pack_rows<bf16>(L, s, reinterpret_cast<bf16*>(dst), D.rows, D.cols, D.dst_ld,
                                         D.row_mult, D.row_off, D.col_off)
                : launch_pack_rows<float>(L, s, reinterpret_cast<float*>(dst), D.rows, D.cols, D.dst_ld,
                                          D.row_mult, D.row_off, D.col_off);
            CK(e);
        }
    }
    m->loaded.insert(n);
    return RLT_OK;
}

rlt_status rlt_model_commit(rlt_model* m) {
    if (!m) return RLT_EINVAL;
    for (const auto& n : m->required)
        if (!m->loaded.count(n)) return RLT_EINVAL;
    m->version += 1;
    return RLT_OK;
}

uint64_t rlt_model_version(const rlt_model* m) { return m ? m->version : 0; }

size_t rlt_encode_workspace_bytes(const rlt_model* m, int B, int T) {
    if (!m || B < 1 || T < 1) return 0;
    return enc_ws(m->cfg, B, T).total;
}

rlt_status rlt_encode(rlt_model* m, const int32_t* tokens, int B, int T, int T_alloc, void* e, void* M,
                      void* ws, size_t ws_bytes, void* stream) {
    if (!m || !tokens || !e || !M || !ws || B < 1 || T < 1 || T > T_alloc || T_alloc > m->cfg.max_pos)
        return RLT_EINVAL;
    if (m->version == 0) return RLT_EINVAL;
    if (!aligned(e) || !aligned(M) || !aligned(ws) || !aligned(tokens, 4)) return RLT_EINVAL;
    if (ws_bytes < enc_ws(m->cfg, B, T).total) return RLT_EINVAL;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* w = reinterpret_cast<uint8_t*>(ws);
    int p = m->prof.begin(RLT_K_ENCODER, st);
    rlt_status s = m->cfg.dtype == RLT_BF16
        ? encode_impl<bf16>(m, tokens, B, T, T_alloc, (bf16*)e, (bf16*)M, w, st)
        : encode_impl<float>(m, tokens, B, T, T_alloc, (float*)e, (float*)M, w, st);
    m->prof.end(p, st);
    return s;
}

size_t rlt_state_bytes(const rlt_model* m, int B) {
    if (!m || B < 1) return 0;
    const rlt_config& c = m->cfg;
    return state_pos_off(c, B) + align_up((size_t)B * 4);
}

rlt_status rlt_state_init(rlt_model* m, void* state, int B, void* stream) {
    if (!m || !state || B < 1 || !aligned(state)) return RLT_EINVAL;
    if (m->version == 0) return RLT_EINVAL;
    rlt_status s = m->cfg.dtype == RLT_BF16
        ? state_init_impl<bf16>(m, (uint8_t*)state, B, (cudaStream_t)stream)
        : state_init_impl<float>(m, (uint8_t*)state, B, (cudaStream_t)stream);
    if (s != RLT_OK) return s;
    m->states[state] = StateInfo::uniform(B, 0, m->version);
    return RLT_OK;
}

rlt_status rlt_state_copy(rlt_model* m, void* dst, const void* src, void* stream) {
    if (!m || !dst || !src || !aligned(dst)) return RLT_EINVAL;
    auto it = m->states.find(src);
    if (it == m->states.end()) return RLT_ESTATE;
    StateInfo info = it->second;
    CK(cudaMemcpyAsync(dst, src, rlt_state_bytes(m, info.B), cudaMemcpyDeviceToDevice,
                       reinterpret_cast<cudaStream_t>(stream)));
    m->states[dst] = info;
    return RLT_OK;
}

rlt_status rlt_state_position(const rlt_model* m, const void* state, int64_t* t) {
    if (!m || !state || !t) return RLT_EINVAL;
    auto it = m->states.find(state);
    if (it == m->states.end()) return RLT_ESTATE;
    *t = it->second.t_max();
    return RLT_OK;
}

rlt_status rlt_state_release(rlt_model* m, const void* state) {
    if (!m || !state) return RLT_EINVAL;
    return m->states.erase(state) ? RLT_OK : RLT_ESTATE;
}

rlt_status rlt_state_positions(const rlt_model* m, const void* state, int64_t* positions) {
    if (!m || !state || !positions) return RLT_EINVAL;
    auto it = m->states.find(state);
    if (it == m->states.end()) return RLT_ESTATE;
    for (size_t b = 0; b < it->second.pos.size(); ++b) positions[b] = it->second.pos[b];
    return RLT_OK;
}

size_t rlt_state_positions_offset(const rlt_model* m, int B) {
    if (!m || B < 1) return 0;
    return state_pos_off(m->cfg, B);
}

rlt_status rlt_state_reset_row(rlt_model* m, void* state, int row, void* stream) {
    if (!m || !state) return RLT_EINVAL;
    auto it = m->states.find(state);
    if (it == m->states.end()) return RLT_ESTATE;
    if (it->second.version != m->version) return RLT_ESTALE;
    const int B = it->second.B;
    if (row < 0 || row >= B) return RLT_EINVAL;
    Launch L = m->launch(stream);
    uint8_t* st = reinterpret_cast<uint8_t*>(state);
    CK(launch_state_init(L, m->at<float>(m->lay.s_star), B, m->cfg.d, reinterpret_cast<float*>(st + state_s_off()),
                         reinterpret_cast<StateHeader*>(st), m->version, state_pos(m->cfg, st, B), row));
    it->second.pos[(size_t)row] = 0;
    return RLT_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- sequence snapshots
namespace {

constexpr uint64_t SNAP_MAGIC = 0x31504e53544c52ull;   // "RLTSNP1"

struct SnapHeader {            // first 256 bytes of a sequence snapshot
    uint64_t magic;
    uint64_t version;          // model version the sequence was built under
    int64_t t;                 // tokens consumed
    int32_t d, n_heads, head_dim, L_E, L_D, W, G, V, dtype, has_enc;
    uint8_t pad[256 - 24 - 40];
};
static_assert(sizeof(SnapHeader) == 256, "snapshot header size");

struct SnapLayout {
    size_t s, ring, mem, enc, total;
};
SnapLayout snap_layout(const rlt_config& c, int64_t t) {
    const size_t e = c.dtype == RLT_BF16 ? 2 : 4, H = c.n_heads, hd = c.head_dim;
    SnapLayout L;
    size_t off = ALIGN;
    auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes); return o; };
    L.s = take((size_t)c.d * 4);
    L.ring = take((size_t)c.L_D * 2 * H * (size_t)(c.W - 1) * hd * e);
    L.mem = take((size_t)c.G * 2 * H * (size_t)t * hd * e);
    L.enc = take((size_t)c.L_E * 2 * H * (size_t)t * hd * e);
    L.total = off;
    return L;
}

// Copy sequence `row`'s blocks between a batch buffer laid out [n_outer][B][H][cap][hd] and a
// snapshot laid out [n_outer][H][t][hd] (to_snap: batch -> snapshot).
cudaError_t copy_rows(uint8_t* snap, uint8_t* batch, int n_outer, int B, int row, int H, int cap, int64_t t, int hd,
                      size_t esz, bool to_snap, cudaStream_t st) {
    if (t <= 0) return cudaSuccess;
    const size_t width = (size_t)t * hd * esz, bpitch = (size_t)cap * hd * esz;
    for (int o = 0; o < n_outer; ++o) {
        uint8_t* sp = snap + (size_t)o * H * width;
        uint8_t* bp = batch + (((size_t)o * B + row) * H) * bpitch;
        cudaError_t e = to_snap ? cudaMemcpy2DAsync(sp, width, bp, bpitch, width, H, cudaMemcpyDeviceToDevice, st)
                                : cudaMemcpy2DAsync(bp, bpitch, sp, width, width, H, cudaMemcpyDeviceToDevice, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

extern "C" {

size_t rlt_snapshot_bytes(const rlt_model* m, int T) {
    if (!m || T < 0) return 0;
    return snap_layout(m->cfg, T).total;
}

rlt_status rlt_snapshot_save(rlt_model* m, const void* state, int row, const void* enc_cache, int T_max,
                             const void* M, int T_alloc, void* dst, size_t dst_bytes, void* stream) {
    if (!m || !state || !M || !dst || !aligned(dst)) return RLT_EINVAL;
    auto it = m->states.find(state);
    if (it == m->states.end()) return RLT_ESTATE;
    const StateInfo& info = it->second;
    if (info.version != m->version) return RLT_ESTALE;
    const int B = info.B;
    if (row < 0 || row >= B) return RLT_EINVAL;
    const rlt_config& c = m->cfg;
    const int64_t t = info.pos[(size_t)row];
    if (t > T_alloc || (enc_cache && t > T_max)) return RLT_EINVAL;
    const SnapLayout S = snap_layout(c, t);
    if (dst_bytes < S.total) return RLT_EINVAL;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* out = reinterpret_cast<uint8_t*>(dst);
    const uint8_t* sb = reinterpret_cast<const uint8_t*>(state);
    const size_t esz = m->lay.esz, H = c.n_heads, hd = c.head_dim;
    SnapHeader h;
    std::memset(&h, 0, sizeof(h));
    h.magic = SNAP_MAGIC; h.version = m->version; h.t = t;
    h.d = c.d; h.n_heads = c.n_heads; h.head_dim = c.head_dim; h.L_E = c.L_E; h.L_D = c.L_D; h.W = c.W; h.G = c.G;
    h.V = c.V; h.dtype = c.dtype; h.has_enc = enc_cache ? 1 : 0;
    CK(cudaMemcpyAsync(out, &h, sizeof(h), cudaMemcpyHostToDevice, st));
    CK(cudaMemcpyAsync(out + S.s, sb + state_s_off() + (size_t)row * c.d * 4, (size_t)c.d * 4,
                       cudaMemcpyDeviceToDevice, st));
    const size_t ring_row = 2 * H * (size_t)(c.W - 1) * hd * esz;
    if (ring_row > 0)
        CK(cudaMemcpy2DAsync(out + S.ring, ring_row, sb + state_ring_off(c, B) + (size_t)row * ring_row, B * ring_row,
                             ring_row, c.L_D, cudaMemcpyDeviceToDevice, st));
    CK(copy_rows(out + S.mem, (uint8_t*)M, 2 * c.G, B, row, c.n_heads, T_alloc, t, hd, esz, true, st));
    if (enc_cache)
        CK(copy_rows(out + S.enc, (uint8_t*)enc_cache, 2 * c.L_E, B, row, c.n_heads, T_max, t, hd, esz, true, st));
    return RLT_OK;
}

rlt_status rlt_snapshot_load(rlt_model* m, const void* src, void* state, int row, void* enc_cache, int T_max,
                             void* M, int T_alloc, void* stream) {
    if (!m || !src || !state || !M || !aligned(src)) return RLT_EINVAL;
    auto it = m->states.find(state);
    if (it == m->states.end()) return RLT_ESTATE;
    StateInfo& info = it->second;
    if (info.version != m->version) return RLT_ESTALE;
    const int B = info.B;
    if (row < 0 || row >= B) return RLT_EINVAL;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    SnapHeader h;
    CK(cudaMemcpyAsync(&h, src, sizeof(h), cudaMemcpyDeviceToHost, st));
    CK(cudaStreamSynchronize(st));
    const rlt_config& c = m->cfg;
    if (h.magic != SNAP_MAGIC || h.d != c.d || h.n_heads != c.n_heads || h.head_dim != c.head_dim ||
        h.L_E != c.L_E || h.L_D != c.L_D || h.W != c.W || h.G != c.G || h.V != c.V || h.dtype != c.dtype)
        return RLT_EINVAL;
    if (h.version != m->version) return RLT_ESTALE;      // built under weights since replaced
    const int64_t t = h.t;
    if (t < 0 || t >= T_alloc || T_alloc > c.max_pos || (enc_cache && (!h.has_enc || t >= T_max))) return RLT_EINVAL;
    const SnapLayout S = snap_layout(c, t);
    const uint8_t* in = reinterpret_cast<const uint8_t*>(src);
    uint8_t* sb = reinterpret_cast<uint8_t*>(state);
    const size_t esz = m->lay.esz, H = c.n_heads, hd = c.head_dim;
    CK(cudaMemcpyAsync(sb + state_s_off() + (size_t)row * c.d * 4, in + S.s, (size_t)c.d * 4,
                       cudaMemcpyDeviceToDevice, st));
    const size_t ring_row = 2 * H * (size_t)(c.W - 1) * hd * esz;
    if (ring_row > 0)
        CK(cudaMemcpy2DAsync(sb + state_ring_off(c, B) + (size_t)row * ring_row, B * ring_row, in + S.ring, ring_row,
                             ring_row, c.L_D, cudaMemcpyDeviceToDevice, st));
    CK(copy_rows(const_cast<uint8_t*>(in) + S.mem, (uint8_t*)M, 2 * c.G, B, row, c.n_heads, T_alloc, t, hd, esz,
                 false, st));
    if (enc_cache)
        CK(copy_rows(const_cast<uint8_t*>(in) + S.enc, (uint8_t*)enc_cache, 2 * c.L_E, B, row, c.n_heads, T_max, t, hd,
                     esz, false, st));
    const int32_t p32 = (int32_t)t;
    CK(cudaMemcpyAsync(state_pos(c, sb, B) + row, &p32, 4, cudaMemcpyHostToDevice, st));
    CK(cudaStreamSynchronize(st));                         // p32 is a host local
    info.pos[(size_t)row] = t;
    return RLT_OK;
}

size_t rlt_decode_workspace_bytes(const rlt_model* m, int B) {
    if (!m || B < 1) return 0;
    return dec_ws(m->cfg, B).total;
}

rlt_status rlt_decode_step(rlt_model* m, void* state, int B, const void* e, const void* M, int T_alloc,
                           const int32_t* next_tok, float tau, float* logp_tok, float* lse, float* logp_full,
                           void* ws, size_t ws_bytes, void* stream) {
    if (!m || !state || !e || !M || !ws || B < 1 || !(tau > 0.f)) return RLT_EINVAL;
    auto it = m->states.find(state);
    if (it == m->states.end() || it->second.B != B) return RLT_ESTATE;
    if (it->second.version != m->version) return RLT_ESTALE;
    int64_t t = it->second.t_max() + 1;           // the furthest sequence's step
    if (t > T_alloc || T_alloc > m->cfg.max_pos) return RLT_EINVAL;
    if (!aligned(e) || !aligned(M) || !aligned(ws)) return RLT_EINVAL;
    if (ws_bytes < dec_ws(m->cfg, B).total) return RLT_EINVAL;
    if ((next_tok && !aligned(next_tok, 4)) || (logp_tok && !aligned(logp_tok, 4)) ||
        (lse && !aligned(lse, 4)) || (logp_full && !aligned(logp_full, 4)))
        return RLT_EINVAL;
    StepIO io;
    io.tok = next_tok; io.logp_tok = next_tok ? logp_tok : nullptr; io.lse = lse; io.logp_full = logp_full;
    io.tau = tau;
    io.head = (next_tok && logp_tok) || lse || logp_full;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    rlt_status s = m->cfg.dtype == RLT_BF16
        ? step_impl<bf16>(m, (uint8_t*)state, B, (const bf16*)e, (const bf16*)M, T_alloc, (int)t, io,
                          (uint8_t*)ws, st)
        : step_impl<float>(m, (uint8_t*)state, B, (const float*)e, (const float*)M, T_alloc, (int)t, io,
                           (uint8_t*)ws, st);
    if (s == RLT_OK)
        for (int64_t& p : it->second.pos) p += 1;
    return s;
}

size_t rlt_encoder_cache_bytes(const rlt_model* m, int B, int T_max) {
    if (!m || B < 1 || T_max < 1) return 0;
    return (size_t)m->cfg.L_E * enc_cache_layer_elems(m->cfg, B, T_max) * m->lay.esz;
}

rlt_status rlt_encode_prefill(rlt_model* m, const int32_t* tokens, int B, int T, int T_alloc, void* e, void* M,
                              void* enc_cache, int T_max, void* ws, size_t ws_bytes, void* stream) {
    if (!m || !tokens || !e || !M || !enc_cache || !ws || B < 1 || T < 1 || T > T_alloc || T_alloc > m->cfg.max_pos)
        return RLT_EINVAL;
    if (T > T_max || T_max > m->cfg.max_pos) return RLT_EINVAL;
    if (m->version == 0) return RLT_EINVAL;
    if (!aligned(e) || !aligned(M) || !aligned(ws) || !aligned(enc_cache) || !aligned(tokens, 4)) return RLT_EINVAL;
    if (ws_bytes < enc_ws(m->cfg, B, T).total) return RLT_EINVAL;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* w = reinterpret_cast<uint8_t*>(ws);
    int p = m->prof.begin(RLT_K_ENCODER, st);
    rlt_status s = m->cfg.dtype == RLT_BF16
        ? encode_impl<bf16>(m, tokens, B, T, T_alloc, (bf16*)e, (bf16*)M, w, st, (bf16*)enc_cache, T_max)
        : encode_impl<float>(m, tokens, B, T, T_alloc, (float*)e, (float*)M, w, st, (float*)enc_cache, T_max);
    m->prof.end(p, st);
    return s;
}

size_t rlt_encode_append_workspace_bytes(const rlt_model* m, int B) {
    if (!m || B < 1) return 0;
    return app_ws(m->cfg, B).total;
}

rlt_status rlt_encode_append(rlt_model* m, const int32_t* tokens, int tok_stride, int B, int pos,
                             const int32_t* positions, void* enc_cache, int T_max, void* e, void* M, int T_alloc,
                             void* ws, size_t ws_bytes, void* stream) {
    if (!m || !tokens || !enc_cache || !e || !M || !ws || B < 1 || tok_stride < 1 || pos < 0) return RLT_EINVAL;
    if (pos >= T_max || pos >= T_alloc || T_max > m->cfg.max_pos || T_alloc > m->cfg.max_pos) return RLT_EINVAL;
    if (m->version == 0) return RLT_EINVAL;
    if (!aligned(e) || !aligned(M) || !aligned(ws) || !aligned(enc_cache) || !aligned(tokens, 4)) return RLT_EINVAL;
    if (positions && !aligned(positions, 4)) return RLT_EINVAL;
    if (ws_bytes < app_ws(m->cfg, B).total) return RLT_EINVAL;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* w = reinterpret_cast<uint8_t*>(ws);
    return m->cfg.dtype == RLT_BF16
        ? encode_append_impl<bf16>(m, tokens, tok_stride, B, pos, positions, (bf16*)enc_cache, T_max, (bf16*)e,
                                   (bf16*)M, T_alloc, w, st)
        : encode_append_impl<float>(m, tokens, tok_stride, B, pos, positions, (float*)enc_cache, T_max, (float*)e,
                                    (float*)M, T_alloc, w, st);
}

rlt_status rlt_sample(rlt_model* m, const float* logp, int B, const float* u, int top_k, float top_p,
                      int32_t* tokens, int tok_stride, float* behaviour_logp, void* stream) {
    if (!m || !logp || !u || !tokens || B < 1 || tok_stride < 1 || top_k < 0 || !(top_p > 0.f) || top_p > 1.f)
        return RLT_EINVAL;
    if (!aligned(logp, 4) || !aligned(u, 4) || !aligned(tokens, 4) || (behaviour_logp && !aligned(behaviour_logp, 4)))
        return RLT_EINVAL;
    if (m->cfg.V > sample_max_vocab()) return RLT_EUNSUPPORTED;
    Launch L = m->launch(stream);
    CK(launch_sample(L, logp, B, m->cfg.V, u, top_k, top_p, tokens, tok_stride, behaviour_logp));
    return RLT_OK;
}

// ---------------------------------------------------------------- decode step without allocation
//
// Scratch for rlt_decode_step_noalloc: a file-scope device array that every GPU which loads
// this library holds until the process exits.  Its device address is looked up once per
// device (cudaGetSymbolAddress with that device current); host code never passes the
// array's host-side name to a kernel.
}  // extern "C"

namespace {
constexpr size_t NOALLOC_SCRATCH_BYTES = size_t(32) << 20;
static __device__ __align__(256) uint8_t g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

constexpr int NOALLOC_MAX_DEVICES = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[NOALLOC_MAX_DEVICES] = {};

rlt_status noalloc_scratch_for_device(int dev, void** out) {
    if (dev < 0 || dev >= NOALLOC_MAX_DEVICES) return RLT_EUNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return RLT_ECUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return RLT_OK;
}
}  // namespace

extern "C" {

rlt_status rlt_decode_step_noalloc(rlt_model* m, void* state, int B, const void* e, const void* M, int T_alloc,
                                   const int32_t* next_tok, float tau, float* logp_tok, float* lse,
                                   float* logp_full, void* stream) {
    if (!m || B < 1) return RLT_EINVAL;
    size_t need = rlt_decode_workspace_bytes(m, B);
    if (need == 0) return RLT_EINVAL;
    if (need > NOALLOC_SCRATCH_BYTES) return RLT_EUNSUPPORTED;   // batch too large for the static scratch
    // the scratch looked up below belongs to the current device: it must be the model's
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return RLT_ECUDA;
    if (dev != m->device) return RLT_EINVAL;
    void* scratch = nullptr;
    rlt_status st = noalloc_scratch_for_device(dev, &scratch);
    if (st != RLT_OK) return st;
    // Every workspace buffer of a step is fully written before it is read, so nothing in the
    // shared scratch has to start at zero.
    return rlt_decode_step(m, state, B, e, M, T_alloc, next_tok, tau, logp_tok, lse, logp_full, scratch,
                           NOALLOC_SCRATCH_BYTES, stream);
}

size_t rlt_replay_workspace_bytes(const rlt_model* m, int B, int T) {
    if (!m || B < 1 || T < 1) return 0;
    const rlt_config& c = m->cfg;
    size_t enc = enc_ws(c, B, T).total, dec = dec_ws(c, B).total;
    return replay_e_bytes(c, B, T) + replay_M_bytes(c, B, T) + rlt_state_bytes(m, B) + (enc > dec ? enc : dec);
}

rlt_status rlt_replay(rlt_model* m, const int32_t* tokens, int B, int T, const int32_t* prompt_len, float tau,
                      float* score, float* logp_tok, void* final_state, void* ws, size_t ws_bytes, void* stream) {
    if (!m || !tokens || !prompt_len || !score || !ws || B < 1 || T < 1 || !(tau > 0.f)) return RLT_EINVAL;
    if (m->version == 0 || T > m->cfg.max_pos) return RLT_EINVAL;
    if (!aligned(ws) || !aligned(tokens, 4) || !aligned(prompt_len, 4) || !aligned(score, 4) ||
        (logp_tok && !aligned(logp_tok, 4)) || (final_state && !aligned(final_state)))
        return RLT_EINVAL;
    if (ws_bytes < rlt_replay_workspace_bytes(m, B, T)) return RLT_EINVAL;
    const rlt_config& c = m->cfg;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* w = reinterpret_cast<uint8_t*>(ws);
    uint8_t* e = w;
    uint8_t* M = e + replay_e_bytes(c, B, T);
    uint8_t* own_state = M + replay_M_bytes(c, B, T);
    uint8_t* scratch = own_state + rlt_state_bytes(m, B);
    uint8_t* state = final_state ? reinterpret_cast<uint8_t*>(final_state) : own_state;
    bool bf = c.dtype == RLT_BF16;
    int p = m->prof.begin(RLT_K_ENCODER, st);
    rlt_status s = bf ? encode_impl<bf16>(m, tokens, B, T, T, (bf16*)e, (bf16*)M, scratch, st)
                      : encode_impl<float>(m, tokens, B, T, T, (float*)e, (float*)M, scratch, st);
    m->prof.end(p, st);
    if (s != RLT_OK) return s;
    s = bf ? state_init_impl<bf16>(m, state, B, st) : state_init_impl<float>(m, state, B, st);
    if (s != RLT_OK) return s;
    CK(cudaMemsetAsync(score, 0, (size_t)B * 4, st));
    if (logp_tok) CK(cudaMemsetAsync(logp_tok, 0, (size_t)B * T * 4, st));
    for (int t = 1; t <= T; ++t) {
        StepIO io;
        io.tau = tau;
        io.head = t < T;
        if (t < T) {
            io.tok = tokens + t;          // x_{t+1} is column t (0-based) of row b
            io.tok_stride = T;
            io.logp_tok = logp_tok ? logp_tok + (t - 1) : nullptr;
            io.lp_stride = T;
            io.score = score;
            io.prompt_len = prompt_len;
        }
        s = bf ? step_impl<bf16>(m, state, B, (const bf16*)e, (const bf16*)M, T, t, io, scratch, st)
               : step_impl<float>(m, state, B, (const float*)e, (const float*)M, T, t, io, scratch, st);
        if (s != RLT_OK) return s;
    }
    if (final_state) m->states[final_state] = StateInfo::uniform(B, T, m->version);
    return RLT_OK;
}

rlt_status rlt_last_error(rlt_model* m, void* stream) {
    if (!m) return RLT_EINVAL;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return RLT_ECUDA;
    uint32_t flags = 0;
    if (cudaMemcpy(&flags, &m->hdr()->err_flags, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return RLT_ECUDA;
    if (flags) {
        uint32_t zero = 0;
        if (cudaMemcpy(&m->hdr()->err_flags, &zero, 4, cudaMemcpyHostToDevice) != cudaSuccess) return RLT_ECUDA;
    }
    if (flags & ERR_TIMEOUT) return RLT_ETIMEOUT;
    if (flags) return RLT_EDEVICE;
    return RLT_OK;
}

uint64_t rlt_launch_count(const rlt_model* m) { return m ? m->launches : 0; }

rlt_status rlt_set_option(rlt_model* m, const char* name, int64_t value) {
    if (!m || !name) return RLT_EINVAL;
    const std::string n(name);
    if (n == "row_groups") {
        if (value < 1 || value > 2) return RLT_EINVAL;
        m->opt_row_groups = (int)value;
    } else if (n == "attn_ctas_per_sm") {
        if (value < 0 || value > 32) return RLT_EINVAL;
        m->opt_attn_cap = (int)value;
    } else if (n == "small_step") {
        if (value < 0 || value > 1) return RLT_EINVAL;
        m->opt_small_step = (int)value;
    } else if (n == "persistent_gemm") {
        if (value < 0 || value > 1) return RLT_EINVAL;
        m->opt_persistent = (int)value;
    } else if (n == "gemv_rows") {
        if (value < 0 || value > 4) return RLT_EINVAL;
        m->opt_gemv_rows = (int)value;
    } else if (n == "group_pdl") {
        if (value < 0 || value > 1) return RLT_EINVAL;
        m->opt_group_pdl = (int)value;
    } else {
        return RLT_EINVAL;
    }
    return RLT_OK;
}

int rlt_gemm_plan(int M, int N, int K) {
    if (M < 1 || N < 1 || K < 1) return -1;
    if (gemm_swap_preferred(M, N, K)) {
        const int s = gemm_swap_auto_split(M, N, K);
        return 11 + (s == 1 ? 1 : (s == 2 ? 2 : (s == 4 ? 3 : 4)));
    }
    return 2 + gemm_tc_pick(M, N, K);
}

rlt_status rlt_gemm_bf16(rlt_model* m, const void* A, const void* W, float* C, int M, int N, int K, int kernel,
                         void* stream) {
    const int n_tc = gemm_tc_variants();
    if (!m || !A || !W || !C || M < 1 || N < 1 || K < 1 || kernel < 0 || kernel > 3 + n_tc + 5 + N_PAIR_VARIANTS)
        return RLT_EINVAL;
    if (kernel > 1 + n_tc && kernel <= 1 + n_tc + 5 && !gemm_swap_supported(M)) return RLT_EINVAL;
    if (kernel == 2 + n_tc + 5 && !gemv_supported(M, N, K, K, A, W)) return RLT_EINVAL;
    if (!aligned(A, 16) || !aligned(W, 16) || !aligned(C, 16) || K % 8 || N % 4) return RLT_EINVAL;
    Launch L = m->launch(stream);
    EpiArgs ea;
    ea.hdr = m->hdr();
    ea.out_f32 = C;
    ea.ld_out = N;
    const bf16* a = reinterpret_cast<const bf16*>(A);
    const bf16* w = reinterpret_cast<const bf16*>(W);
    if (kernel == 0) {
        CK(launch_gemm<bf16>(L, Epi::StoreF32, a, K, w, M, N, K, ea));
    } else if (kernel == 1) {
        CK(launch_gemm_simt<bf16>(L, Epi::StoreF32, a, K, w, M, N, K, ea));
    } else if (kernel <= 1 + n_tc) {
        CK(launch_gemm_tc(L, Epi::StoreF32, a, K, w, M, N, K, ea, m->hdr(), kernel - 2));
    } else if (kernel <= 1 + n_tc + 5) {
        static const int splits[5] = {0, 1, 2, 4, 8};
        CK(launch_gemm_swap(L, Epi::StoreF32, a, K, w, M, N, K, ea, m->hdr(), splits[kernel - 2 - n_tc]));
    } else if (kernel == 2 + n_tc + 5) {
        CK(launch_gemv(L, Epi::StoreF32, a, K, w, M, N, K, ea, m->hdr()));
    } else if (kernel == 3 + n_tc + 5) {
        CK(launch_gemm_tc(L, Epi::StoreF32, a, K, w, M, N, K, ea, m->hdr(), PERSISTENT_VARIANT));
    } else {
        CK(launch_gemm_tc(L, Epi::StoreF32, a, K, w, M, N, K, ea, m->hdr(), PAIR_VARIANT + kernel - (4 + n_tc + 5)));
    }
    return RLT_OK;
}

rlt_status rlt_selftest_wait_timeout(rlt_model* m, const void* A, const void* W, float* C, int M, int N, int K,
                                     int kernel, uint64_t wait_ns, void* stream) {
    const int n_tc = gemm_tc_variants();
    const int pair0 = 4 + n_tc + 5;          // kernel ids of the CTA-pair tiles
    const bool pair = kernel >= pair0 && kernel < pair0 + N_PAIR_VARIANTS;
    if (!m || !A || !W || !C || M < 1 || N < 1 || K < 1 || kernel < 2 || (kernel > 1 + n_tc + 5 && !pair))
        return RLT_EINVAL;
    if (kernel > 1 + n_tc && !pair && !gemm_swap_supported(M)) return RLT_EINVAL;
    if (!aligned(A, 16) || !aligned(W, 16) || !aligned(C, 16) || K % 8 || N % 4) return RLT_EINVAL;
    if (wait_ns < 1000 || wait_ns > 2000000000ull) return RLT_EINVAL;
    Launch L = m->launch(stream);
    EpiArgs ea;
    ea.hdr = m->hdr();
    ea.out_f32 = C;
    ea.ld_out = N;
    ea.wait_ns = wait_ns;
    ea.no_loads = 1;
    const bf16* a = reinterpret_cast<const bf16*>(A);
    const bf16* w = reinterpret_cast<const bf16*>(W);
    if (pair) {
        CK(launch_gemm_tc(L, Epi::StoreF32, a, K, w, M, N, K, ea, m->hdr(), PAIR_VARIANT + kernel - pair0));
    } else if (kernel <= 1 + n_tc) {
        CK(launch_gemm_tc(L, Epi::StoreF32, a, K, w, M, N, K, ea, m->hdr(), kernel - 2));
    } else {
        static const int splits[5] = {0, 1, 2, 4, 8};
        CK(launch_gemm_swap(L, Epi::StoreF32, a, K, w, M, N, K, ea, m->hdr(), splits[kernel - 2 - n_tc]));
    }
    return RLT_OK;
}

rlt_status rlt_profile_start(rlt_model* m, uint32_t kind_mask) {
    if (!m) return RLT_EINVAL;
    m->prof.on = true;
    m->prof.mask = kind_mask;
    m->prof.used = 0;
    m->prof.recs.clear();
    return RLT_OK;
}

rlt_status rlt_profile_stop(rlt_model* m, double* ms, uint64_t* launches) {
    if (!m) return RLT_EINVAL;
    Profiler& P = m->prof;
    P.on = false;
    if (ms) for (int k = 0; k < RLT_K_COUNT; ++k) ms[k] = 0.0;
    if (launches) for (int k = 0; k < RLT_K_COUNT; ++k) launches[k] = 0;
    if (P.used && cudaEventSynchronize(P.pool[P.used - 1]) != cudaSuccess) return RLT_ECUDA;
    for (const auto& r : P.recs) {
        float e = 0.f;
        if (cudaEventElapsedTime(&e, P.pool[r.second], P.pool[r.second + 1]) != cudaSuccess) return RLT_ECUDA;
        if (ms) ms[r.first] += e;
        if (launches) launches[r.first] += 1;
    }
    P.recs.clear();
    P.used = 0;
    return RLT_OK;
}

}  // extern "C"
