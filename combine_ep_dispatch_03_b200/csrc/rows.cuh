// rows.cuh -- per-element work shared by the row movers: bf16 unpacking and
// round-to-nearest-even packing, the e4m3 cast, and the FP8 block cast of a
// 16-element chunk (per-128-element scale amax / 448, NCCL EP paper Table IV).
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "fast_div.cuh"

namespace epb {

__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

__device__ __forceinline__ void unpack8(const uint4 &v, float *f) {
    f[0] = bf16lo(v.x); f[1] = bf16hi(v.x);
    f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
    f[4] = bf16lo(v.z); f[5] = bf16hi(v.z);
    f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}

// round-to-nearest-even to bf16, two at a time (lo -> low half)
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

__device__ __forceinline__ uint4 pack8(const float *f) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                      pack_bf16x2(f[6], f[7]));
}

// e4m3 with round-to-nearest-even and saturation to +-448; `lo` lands in the
// low byte (the element at the lower address).
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// One 16-element chunk (two 16-byte halves of bf16) to 16 e4m3 codes and its
// block's scale. Every lane of the warp calls it at once: the block's amax is
// reduced over the 8 lanes holding the block.
__device__ __forceinline__ void quant_chunk(const uint4 &a, const uint4 &b, uint4 &q, float &sc) {
    float f[16];
    unpack8(a, f);
    unpack8(b, f + 8);
    float amax = 0.0f;
#pragma unroll
    for (int u = 0; u < 16; ++u) amax = fmaxf(amax, fabsf(f[u]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
    const float s = __fdiv_rn(amax, 448.0f);
    sc = s;
    uint32_t wd[4] = {0u, 0u, 0u, 0u};
    if (amax != 0.0f) {
        const float y = __frcp_rn(s);
        float minnz = INFINITY;
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const float m = fabsf(f[u]);
            minnz = fminf(minnz, m > 0.0f ? m : INFINITY);
        }
        if (fast_group_ok(amax, minnz, y)) {
#pragma unroll
            for (int u = 0; u < 16; ++u) f[u] = div_by_scale_fast(f[u], s, y);
        } else {
#pragma unroll
            for (int u = 0; u < 16; ++u) f[u] = __fdiv_rn(f[u], s);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) wd[u] = e4m3x2(f[4 * u], f[4 * u + 1]) | (e4m3x2(f[4 * u + 2], f[4 * u + 3]) << 16);
    }
    q = make_uint4(wd[0], wd[1], wd[2], wd[3]);
}

// read_before_wait: a dispatch reads its token row x[t] before
// griddepcontrol.wait. The kernels that may run concurrently with that read
// are the routing kernels of the plan just before it (they write routing state
// only, never x) and, through them, nothing older: each routing kernel lets its
// dependents start only after its own wait, that is after every earlier kernel
// of the stream has completed. A caller that writes x with a kernel of its own
// that triggers its dependents early must write x before the trigger.
template <int VPT>
__device__ __forceinline__ void load_slab(const uint4 *__restrict__ src, int c0, int nvec, uint4 *v) {
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int c = c0 + threadIdx.x + i * blockDim.x;
        if (c < nvec) v[i] = __ldcs(src + c);
    }
}

// the two 16-byte halves of each thread's 16-element chunks (zeros past the row)
template <int CPT>
__device__ __forceinline__ void load_pairs(const uint4 *__restrict__ src, int c0, int nchunk, uint4 *a, uint4 *b) {
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int c = c0 + threadIdx.x + i * blockDim.x;
        if (c < nchunk) {
            a[i] = __ldcs(src + 2 * c);
            b[i] = __ldcs(src + 2 * c + 1);
        } else {
            a[i] = make_uint4(0, 0, 0, 0);
            b[i] = a[i];
        }
    }
}

} // namespace epb
