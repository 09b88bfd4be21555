// router.cu -- ep_router_topk: the gating step just before dispatch. For each
// token, the K experts with the largest logits and their router weights
// (softmax over the logits, renormalised over the K chosen experts).
//
// "Ultra-Large MoE Models: Open-Source Evolution and Heterogeneous Inference
// Adaptation", §2.1 (the gating network picks the top-K experts per token)
// and §3.1 (the top-K routing operator, a fused MoE-specific operator).
//
// One warp per token. Lane l holds the logits of experts l, l+32, ..., sorted
// largest first; each of the K rounds is two warp reductions (redux.sync): the
// largest head over the warp, then the lowest id among the lanes holding it
// (ties go to the lower expert id); that lane pops its head. The weights are
// exp(l_k - l_max) / sum_j exp(l_j - l_max) in fp32, summed in k order.
#include "ep_internal.cuh"

namespace epb {
namespace {

constexpr int kRouterWarps = 8;

// Order-preserving map of a finite float to a 32-bit key (larger value ->
// larger key); -0 is taken as +0 so that equal values compare equal. Real keys
// are never 0, which marks an empty candidate.
__device__ __forceinline__ uint32_t order_key(float v) {
    const uint32_t u = __float_as_uint(v == 0.0f ? 0.0f : v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

template <int EPL> // experts per lane: E <= 32 * EPL
__global__ void __launch_bounds__(kRouterWarps * 32) k_router_topk(const float *__restrict__ logits, int T, int E,
                                                                    int K, int32_t *__restrict__ idx,
                                                                    float *__restrict__ w) {
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * kRouterWarps + (threadIdx.x >> 5);
    if (t >= T) return; // whole warp
    const float *l = logits + (int64_t)t * E;
    uint32_t key[EPL];
    int id[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        key[i] = e < E ? order_key(__ldcs(l + e)) : 0u;
        id[i] = e;
    }
    // sort this lane's candidates, largest first; swapping only on a strict
    // inequality keeps equal keys in ascending id order
#pragma unroll
    for (int r = 0; r < EPL; ++r) {
#pragma unroll
        for (int i = r & 1; i + 1 < EPL; i += 2) {
            if (key[i + 1] > key[i]) {
                const uint32_t tk = key[i];
                key[i] = key[i + 1];
                key[i + 1] = tk;
                const int ti = id[i];
                id[i] = id[i + 1];
                id[i + 1] = ti;
            }
        }
    }
    // K rounds: the largest head key over the warp, then the lowest id among
    // the lanes holding it; that lane pops its head
    float my_v = 0.0f; // lane k keeps the k-th choice
    int my_e = -1;
    for (int k = 0; k < K; ++k) {
        const uint32_t m = __reduce_max_sync(0xffffffffu, key[0]);
        const uint32_t cand = key[0] == m ? (uint32_t)id[0] : 0xffffffffu;
        const uint32_t win = __reduce_min_sync(0xffffffffu, cand);
        if (lane == k) {
            my_v = key_value(m);
            my_e = (int)win;
        }
        if (cand == win) {
#pragma unroll
            for (int i = 0; i + 1 < EPL; ++i) {
                key[i] = key[i + 1];
                id[i] = id[i + 1];
            }
            key[EPL - 1] = 0u;
        }
    }
    const float vmax = __shfl_sync(0xffffffffu, my_v, 0);
    const float ex = lane < K ? expf(my_v - vmax) : 0.0f;
    float sum = 0.0f;
    for (int k = 0; k < K; ++k) sum = __fadd_rn(sum, __shfl_sync(0xffffffffu, ex, k)); // fixed k order
    if (lane < K) {
        idx[(int64_t)t * K + lane] = my_e;
        w[(int64_t)t * K + lane] = __fdiv_rn(ex, sum);
    }
}

} // namespace
} // namespace epb

using namespace epb;

extern "C" ep_status_t ep_router_topk(const float *logits, int32_t num_tokens, int32_t num_experts, int32_t topk,
                                      int32_t *topk_idx, float *topk_w, void *stream) {
    const int T = num_tokens, E = num_experts, K = topk;
    if (T < 0 || E < 1 || E > kRouterMaxExperts || K < 1 || K > E || K > kMaxTopk) return EP_ERR_INVALID_ARG;
    if (T == 0) return EP_OK;
    if (!logits || !topk_idx || !topk_w || ((uintptr_t)logits & 3) || ((uintptr_t)topk_idx & 3) ||
        ((uintptr_t)topk_w & 3))
        return EP_ERR_INVALID_ARG;
    const dim3 grid((T + kRouterWarps - 1) / kRouterWarps), block(kRouterWarps * 32);
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t err;
    const int epl = (E + 31) / 32;
    if (epl <= 1)
        err = launch_pdl(k_router_topk<1>, grid, block, 0, st, logits, T, E, K, topk_idx, topk_w);
    else if (epl <= 2)
        err = launch_pdl(k_router_topk<2>, grid, block, 0, st, logits, T, E, K, topk_idx, topk_w);
    else if (epl <= 4)
        err = launch_pdl(k_router_topk<4>, grid, block, 0, st, logits, T, E, K, topk_idx, topk_w);
    else if (epl <= 8)
        err = launch_pdl(k_router_topk<8>, grid, block, 0, st, logits, T, E, K, topk_idx, topk_w);
    else if (epl <= 16)
        err = launch_pdl(k_router_topk<16>, grid, block, 0, st, logits, T, E, K, topk_idx, topk_w);
    else
        err = launch_pdl(k_router_topk<32>, grid, block, 0, st, logits, T, E, K, topk_idx, topk_w);
    return err == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}
