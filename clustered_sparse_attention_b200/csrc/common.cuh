// common.cuh -- small device helpers shared by the library's kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "svgear.h"

namespace svgear {

constexpr int kWarp = 32;

// ---------------------------------------------------------------------------
// Element access: token tensors are float or bfloat16; everything is
// computed in fp32.  A "chunk" is the 16 bytes one lane moves per load.
// ---------------------------------------------------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
    static constexpr int kPerChunk = 4;
    __device__ static inline void load(const float* p, float* out) {
        float4 v = __ldg(reinterpret_cast<const float4*>(p));
        out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
    }
    // one 16-byte chunk kept packed (fewer live registers), unpacked at use
    __device__ static inline uint4 load_raw(const float* p) {
        return __ldg(reinterpret_cast<const uint4*>(p));
    }
    __device__ static inline void unpack(const uint4& v, float* out) {
        out[0] = __uint_as_float(v.x); out[1] = __uint_as_float(v.y);
        out[2] = __uint_as_float(v.z); out[3] = __uint_as_float(v.w);
    }
    __device__ static inline float from(float x) { return x; }
    __device__ static inline float to(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
    static constexpr int kPerChunk = 8;
    __device__ static inline void load(const __nv_bfloat16* p, float* out) {
        uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            out[2 * i] = __uint_as_float(w[i] << 16);
            out[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
    __device__ static inline uint4 load_raw(const __nv_bfloat16* p) {
        return __ldg(reinterpret_cast<const uint4*>(p));
    }
    __device__ static inline void unpack(const uint4& v, float* out) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            out[2 * i] = __uint_as_float(w[i] << 16);
            out[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
    __device__ static inline float from(__nv_bfloat16 x) { return __bfloat162float(x); }
    __device__ static inline __nv_bfloat16 to(float x) { return __float2bfloat16_rn(x); }
};

// Float <-> order-preserving unsigned key (larger float -> larger key).
__device__ inline uint32_t float_to_ordered(float f) {
    uint32_t b = __float_as_uint(f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ inline float ordered_to_float(uint32_t k) {
    uint32_t b = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
    return __uint_as_float(b);
}

__device__ inline float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ---------------------------------------------------------------------------
// Philox4x64-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As
// Easy as 1, 2, 3", SC'11): ten rounds of two 64x64->128 multiplies of the
// even counter words, XOR of the high halves into the odd words and the key,
// with the key bumped by the Weyl constants between rounds.
// ---------------------------------------------------------------------------
__device__ inline void philox4x64_10(uint64_t x[4], uint64_t k0, uint64_t k1) {
    const uint64_t M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
    const uint64_t W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        uint64_t hi0 = __umul64hi(M0, x[0]), lo0 = M0 * x[0];
        uint64_t hi1 = __umul64hi(M1, x[2]), lo1 = M1 * x[2];
        uint64_t y0 = hi1 ^ x[1] ^ k0, y2 = hi0 ^ x[3] ^ k1;
        x[0] = y0; x[1] = lo1; x[2] = y2; x[3] = lo0;
        k0 += W0; k1 += W1;
    }
}

// Uniform double in [0, 1): draw j of stream s under seed (counter
// {j, s, 0, 0}, key {seed, 0}, top 53 bits of the first output word).
__device__ inline double philox_uniform(uint64_t seed, uint64_t stream, uint64_t j) {
    uint64_t x[4] = {j, stream, 0, 0};
    philox4x64_10(x, seed, 0);
    return (double)(x[0] >> 11) * (1.0 / 9007199254740992.0);
}

}  // namespace svgear

namespace svgear {
// Host-side count of kernels this library has launched (all devices).
void count_launches(unsigned n);
}  // namespace svgear

// Launch-error helper for the host side.
#define SVGEAR_LAUNCH_CHECK()                                  \
    do {                                                       \
        if (cudaPeekAtLastError() != cudaSuccess) return SVGEAR_ERR_CUDA; \
    } while (0)
