// Token sampler of the generation loop: one CTA per sequence draws the next token from its
// log-probability row at the sampling temperature, after top-k / top-p truncation, by inverse
// CDF with a caller-given uniform, and returns the behaviour log-probability of the draw (the
// log-probability under the truncated, renormalised distribution actually sampled from).
//
// Truncation keeps every token tied at a boundary: top-k keeps token i when fewer than k
// tokens are strictly more probable; top-p then keeps i when the mass of the strictly more
// probable tokens is below top_p times the mass top-k kept.  With p >= 0 the float bit
// patterns order like the values, so both rules become thresholds on the bit pattern:
//   top-k   the k-th largest pattern, found by a 4-pass radix select (8-bit digits);
//   top-p   the smallest pattern b with mass(pattern > b) < top_p * Z1, found by bisection.
// The kept tokens are then scanned in id order (float64 sums) and the first id whose
// cumulative kept mass exceeds u * Z is the draw.
#include "kernels.cuh"

namespace rlt {

namespace {

constexpr int ST = 1024;            // threads per row
constexpr int SW = ST / 32;

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Sum over the block (every thread gets the total).  `red` holds SW doubles.
__device__ __forceinline__ double block_sum_d(double v, double* red) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    v = warp_sum_d(v);
    __syncthreads();                         // red is free (a previous call may still read it)
    if (lane == 0) red[w] = v;
    __syncthreads();
    double t = lane < SW ? red[lane] : 0.0;
    return warp_sum_d(t);
}

__global__ void __launch_bounds__(ST) k_sample(const float* __restrict__ logp, int V, const float* __restrict__ u,
                                               int top_k, float top_p, int32_t* tok, int tok_stride, float* blp) {
    extern __shared__ uint32_t bits[];       // V patterns of p = exp(logp)
    __shared__ int hist[256];
    __shared__ double red[SW];
    __shared__ int sel_digit, sel_rem, found;
    __shared__ double scan[SW];
    pdl_wait();
    pdl_trigger();
    const int b = blockIdx.x;
    const float* row = logp + (long long)b * V;
    for (int i = threadIdx.x; i < V; i += ST) bits[i] = __float_as_uint(expf(row[i]));
    __syncthreads();

    // top-k: pattern of the k-th largest p (0 keeps everything)
    uint32_t thr = 0;
    if (top_k > 0 && top_k < V) {
        uint32_t prefix = 0, mask = 0;
        int rem = top_k;
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int i = threadIdx.x; i < 256; i += ST) hist[i] = 0;
            __syncthreads();
            for (int i = threadIdx.x; i < V; i += ST) {
                const uint32_t x = bits[i];
                if ((x & mask) == prefix) atomicAdd(&hist[(x >> shift) & 255u], 1);
            }
            __syncthreads();
            if (threadIdx.x == 0) {
                int cum = 0, dg = 0;
                for (dg = 255; dg > 0; --dg) {
                    if (cum + hist[dg] >= rem) break;
                    cum += hist[dg];
                }
                sel_digit = dg;
                sel_rem = rem - cum;
            }
            __syncthreads();
            prefix |= (uint32_t)sel_digit << shift;
            mask |= 255u << shift;
            rem = sel_rem;
        }
        thr = prefix;
    }

    // top-p: the smallest pattern b with mass(pattern > b) < top_p * Z1
    if (top_p < 1.0f) {
        double z1 = 0.0;
        for (int i = threadIdx.x; i < V; i += ST)
            if (bits[i] >= thr) z1 += (double)__uint_as_float(bits[i]);
        z1 = block_sum_d(z1, red);
        const double target = (double)top_p * z1;
        uint32_t lo = 0, hi = 0x7f800000u;
        while (lo < hi) {
            const uint32_t mid = lo + (hi - lo) / 2;
            double above = 0.0;
            for (int i = threadIdx.x; i < V; i += ST)
                if (bits[i] > mid) above += (double)__uint_as_float(bits[i]);
            above = block_sum_d(above, red);
            if (above < target) hi = mid; else lo = mid + 1;
        }
        if (lo > thr) thr = lo;
    }

    // inverse CDF over the kept tokens in id order: thread k scans ids [c0, c1)
    const int per = (V + ST - 1) / ST;
    const int c0 = min(V, (int)threadIdx.x * per), c1 = min(V, c0 + per);
    double local = 0.0;
    for (int i = c0; i < c1; ++i)
        if (bits[i] >= thr) local += (double)__uint_as_float(bits[i]);
    // exclusive scan of the per-thread sums
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    double incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        double y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) scan[w] = incl;
    if (threadIdx.x == 0) found = -1;
    __syncthreads();
    double wbase = 0.0, total = 0.0;
    for (int j = 0; j < SW; ++j) {
        if (j < w) wbase += scan[j];
        total += scan[j];
    }
    const double excl = wbase + incl - local;
    const double r = (double)u[b] * total;
    if (local > 0.0 && excl <= r && r < excl + local) {
        double acc = excl;
        int pick = -1, last = -1;
        for (int i = c0; i < c1; ++i) {
            if (bits[i] < thr) continue;
            acc += (double)__uint_as_float(bits[i]);
            last = i;
            if (acc > r) { pick = i; break; }
        }
        atomicMax(&found, pick >= 0 ? pick : last);
    }
    __syncthreads();
    if (found < 0) {
        // r at or past the total by rounding: the last kept id
        int last = -1;
        for (int i = c1 - 1; i >= c0; --i)
            if (bits[i] >= thr) { last = i; break; }
        if (last >= 0) atomicMax(&found, last);
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const int x = found >= 0 ? found : 0;        // a kept set is never empty; guards a NaN u
        tok[(long long)b * tok_stride] = x;
        if (blp) blp[b] = (float)((double)row[x] - log(total));
    }
}

}  // namespace

int sample_max_vocab() { return 49152; }

cudaError_t launch_sample(Launch L, const float* logp, int B, int V, const float* u, int top_k, float top_p,
                          int32_t* tok, int tok_stride, float* blp) {
    const size_t smem = (size_t)V * 4;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(k_sample, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             sample_max_vocab() * 4);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    return launch_k(L, k_sample, (unsigned)B, ST, smem, logp, V, u, top_k, top_p, tok, tok_stride, blp);
}

}  // namespace rlt
