// The bounded mbarrier wait of bulk.cuh, run on one thread of one CTA:
//   phase 0 is armed by a real 1 KB bulk copy: the wait must succeed and the
//           bytes must arrive;
//   phase 1 is armed for 16 bytes that no copy ever delivers: the wait must
//           give up once its limit has passed.
// Nothing is in flight when the kernel returns. Usage: mbar_timeout <limit_ms>
// or mbar_timeout default (the 2 s limit the dispatch uses). Prints
//   copy_ok C data_ok D gave_up G waited_ns N limit_ns L
// and exits 0 unless a CUDA call failed. Built and run by
// test_mbar_timeout_gpu.py.
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include <cuda_runtime.h>

#include "bulk.cuh"

using namespace epb;

__global__ void probe(const uint4 *src, uint4 *dst, uint64_t limit_ns, int use_default,
                      unsigned long long *out) {
    __shared__ __align__(128) uint4 buf[64];
    __shared__ __align__(8) uint64_t bar;
    mbar_init(&bar);
    bulk_load(buf, src, (uint32_t)sizeof buf, &bar);
    out[0] = mbar_wait(&bar, 0, limit_ns) ? 1ull : 0ull;
    for (int i = 0; i < 64; ++i) dst[i] = buf[i];
    mbar_expect_tx(&bar, 16); // phase 1: nothing will deliver these bytes
    const uint64_t t0 = global_ns();
    const bool done = use_default ? mbar_wait(&bar, 1) : mbar_wait(&bar, 1, limit_ns);
    out[2] = global_ns() - t0;
    out[1] = done ? 0ull : 1ull;
}

int main(int argc, char **argv) {
    if (argc != 2) {
        fprintf(stderr, "usage: %s <limit_ms>|default\n", argv[0]);
        return 2;
    }
    const int use_default = strcmp(argv[1], "default") == 0;
    const uint64_t limit_ns = use_default ? kWaitLimitNs : (uint64_t)atoll(argv[1]) * 1000000ull;
    uint4 host[64], back[64];
    for (int i = 0; i < 64; ++i) host[i] = make_uint4(4 * i, 4 * i + 1, 4 * i + 2, 0x9e3779b9u ^ i);
    uint4 *src = nullptr, *dst = nullptr;
    unsigned long long *out = nullptr, res[3] = {0, 0, 0};
    if (cudaMalloc(&src, sizeof host) != cudaSuccess || cudaMalloc(&dst, sizeof host) != cudaSuccess ||
        cudaMalloc(&out, sizeof res) != cudaSuccess) {
        printf("cuda malloc failed\n");
        return 3;
    }
    cudaMemcpy(src, host, sizeof host, cudaMemcpyHostToDevice);
    cudaMemset(dst, 0, sizeof host);
    cudaMemset(out, 0, sizeof res);
    probe<<<1, 1>>>(src, dst, limit_ns, use_default, out);
    const cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        printf("cuda error %s\n", cudaGetErrorString(e));
        return 4;
    }
    cudaMemcpy(back, dst, sizeof back, cudaMemcpyDeviceToHost);
    cudaMemcpy(res, out, sizeof res, cudaMemcpyDeviceToHost);
    const int data_ok = memcmp(host, back, sizeof host) == 0;
    printf("copy_ok %llu data_ok %d gave_up %llu waited_ns %llu limit_ns %llu\n", res[0], data_ok, res[1], res[2],
           (unsigned long long)limit_ns);
    cudaFree(src);
    cudaFree(dst);
    cudaFree(out);
    return 0;
}
