// Shared device helpers for the RLT library: storage types, 16-byte vector access,
// device error flags and launch bookkeeping.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace rlt {

typedef __nv_bfloat16 bf16;

// Device-side error flags, latched in the model header and read by rlt_last_error.
enum : uint32_t {
    ERR_BAD_TOKEN = 1u,     // a token id outside [0, V)
    ERR_STATE_MISMATCH = 2u,// a state header disagreed with its registered position/version
    ERR_TIMEOUT = 4u,       // a bounded device wait gave up
};

struct DevHeader {          // first 256 bytes of the weight arena
    uint32_t err_flags;
    uint32_t pad0;
    uint64_t version;
    uint8_t pad[240];
};

struct StateHeader {        // first 256 bytes of a decoder state
    uint64_t magic;
    int64_t t;              // tokens consumed
    uint64_t version;       // model version the state was built under
    int32_t B;
    int32_t pad0;
    uint8_t pad[224];
};
static_assert(sizeof(DevHeader) == 256, "header size");
static_assert(sizeof(StateHeader) == 256, "header size");

constexpr uint64_t STATE_MAGIC = 0x524c545354415445ull;   // "RLTSTATE"

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(bf16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }

// Round a float to the storage type and back (the bf16 storage contract).
template <typename T> __device__ __forceinline__ float round_to(float x) { return to_f(from_f<T>(x)); }

// 16 bytes of storage-type elements <-> float registers.
template <typename T> struct Vec16;

template <> struct Vec16<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void unpack(const uint4& r, float* o) {
        o[0] = __uint_as_float(r.x); o[1] = __uint_as_float(r.y);
        o[2] = __uint_as_float(r.z); o[3] = __uint_as_float(r.w);
    }
    __device__ __forceinline__ static uint4 pack(const float* v) {
        return make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]),
                          __float_as_uint(v[2]), __float_as_uint(v[3]));
    }
};

template <> struct Vec16<bf16> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void unpack(const uint4& r, float* o) {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            o[2 * i] = __uint_as_float(w[i] << 16);
            o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ __forceinline__ static uint4 pack(const float* v) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 p = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t*>(&p);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};

__device__ __forceinline__ uint4 ld16(const void* p) { return *reinterpret_cast<const uint4*>(p); }
// streaming load: data read once per pass, not worth keeping in L1
__device__ __forceinline__ uint4 ld16_stream(const void* p) { return __ldcs(reinterpret_cast<const uint4*>(p)); }
__device__ __forceinline__ void st16(void* p, const uint4& v) { *reinterpret_cast<uint4*>(p) = v; }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ void raise_flag(DevHeader* h, uint32_t f) { atomicOr(&h->err_flags, f); }

// Programmatic dependent launch.  Every kernel of the library is launched so that it may
// start while its predecessor on the stream drains; it must call pdl_wait() before it reads
// anything an earlier kernel wrote or writes anything an earlier kernel reads.  pdl_trigger()
// lets the next kernel on the stream be scheduled early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + expf(-x)); }
__device__ __forceinline__ float siluf_(float x) { return x / (1.0f + expf(-x)); }

}  // namespace rlt
