// Exhaustive check of div_by_scale_fast (fast_div.cuh) against __fdiv_rn:
// every positive finite bf16 amax and every finite bf16 x with |x| <= amax,
// scale s = RN(amax / 448) as the FP8 cast forms it. Wherever fast_group_ok
// admits x (as a group of one), the two quotients must have the same bits.
// Prints the counts; exits 0 only if none differs. Built and run by
// test_fast_div_gpu.py.
#include <cstdint>
#include <cstdio>

#include <cuda_runtime.h>

#include "fast_div.cuh"

using namespace epb;

__device__ unsigned long long g_pairs, g_fast, g_mismatch;
__device__ uint32_t g_first[4]; // x, amax, expected, got of one mismatch

__global__ void check(int amax_lo, int amax_hi) {
    const int xb = blockIdx.x * blockDim.x + threadIdx.x; // every 16-bit pattern of x
    if (xb >= 65536) return;
    const float x = __uint_as_float((uint32_t)xb << 16);
    if (!isfinite(x)) return;
    unsigned long long pairs = 0, fast = 0, bad = 0;
    for (int ab = amax_lo; ab < amax_hi; ++ab) {
        const float amax = __uint_as_float((uint32_t)ab << 16);
        if (!(amax > 0.0f) || !isfinite(amax) || fabsf(x) > amax) continue;
        ++pairs;
        const float s = __fdiv_rn(amax, 448.0f);
        const float y = __frcp_rn(s);
        if (!fast_group_ok(amax, x != 0.0f ? fabsf(x) : INFINITY, y)) continue;
        ++fast;
        const float want = __fdiv_rn(x, s), got = div_by_scale_fast(x, s, y);
        if (__float_as_uint(want) != __float_as_uint(got)) {
            ++bad;
            if (atomicCAS(&g_first[0], 0u, __float_as_uint(x) | 1u) == 0u) {
                g_first[1] = __float_as_uint(amax);
                g_first[2] = __float_as_uint(want);
                g_first[3] = __float_as_uint(got);
            }
        }
    }
    atomicAdd(&g_pairs, pairs);
    atomicAdd(&g_fast, fast);
    atomicAdd(&g_mismatch, bad);
}

int main() {
    const int kEnd = 0x7f80; // first non-finite positive bf16 pattern
    for (int lo = 1; lo < kEnd; lo += 512) {
        check<<<256, 256>>>(lo, lo + 512 < kEnd ? lo + 512 : kEnd);
        const cudaError_t e = cudaDeviceSynchronize();
        if (e != cudaSuccess) {
            printf("cuda error: %s\n", cudaGetErrorString(e));
            return 2;
        }
    }
    unsigned long long pairs = 0, fast = 0, bad = 0;
    uint32_t first[4] = {0, 0, 0, 0};
    cudaMemcpyFromSymbol(&pairs, g_pairs, sizeof pairs);
    cudaMemcpyFromSymbol(&fast, g_fast, sizeof fast);
    cudaMemcpyFromSymbol(&bad, g_mismatch, sizeof bad);
    cudaMemcpyFromSymbol(first, g_first, sizeof first);
    printf("pairs %llu fast %llu mismatches %llu\n", pairs, fast, bad);
    if (bad) printf("first mismatch: x~%08x amax=%08x want=%08x got=%08x\n", first[0], first[1], first[2], first[3]);
    return bad == 0 ? 0 : 1;
}
