// router.cu -- ep_router_topk: the gating step just before dispatch. For each
// token, the K experts with the largest logits and their router weights
// (softmax over the logits, renormalised over the K chosen experts).
//
// "Ultra-Large MoE Models: Open-Source Evolution and Heterogeneous Inference
// Adaptation", §2.1 (the gating network picks the top-K experts per token)
// and §3.1 (the top-K routing operator, a fused MoE-specific operator).
//
// One warp per token. Lane l holds experts l, l+32, ..., each as one 32-bit
// word: the logit's order-preserving key with its low bits replaced by the
// inverted expert id, so that one unsigned maximum finds the largest logit and,
// among equal ones, the lowest id (ties go to the lower expert id). Each lane
// sorts its words largest first; each of the K rounds is one warp reduction
// (redux.sync), after which the lane holding the winner pops it. Replacing the
// low key bits can swap two candidates whose keys agree above them; two warp
// votes find every case where that could change the result, and such warps
// redo the selection with full keys and a second reduction per round. The
// weights are exp(l_k - l_max) / sum_j exp(l_j - l_max) in fp32 from the
// chosen logits, summed in k order.
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

// bits of the expert id packed under the key: ids are below 32 * EPL
__host__ __device__ constexpr int id_bits(int epl) { return epl <= 1 ? 5 : epl <= 2 ? 6 : epl <= 4 ? 7 : epl <= 8 ? 8 : epl <= 16 ? 9 : 10; }

// The exact selection, for warps whose packed keys may have reordered two
// candidates: full keys and ids side by side, two warp reductions a round.
// Returns the id of lane k's choice for lanes k < K, else -1.
template <int EPL>
__device__ __noinline__ int topk_exact(const float *__restrict__ l, int lane, int E, int K) {
    uint32_t key[EPL];
    int id[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        key[i] = e < E ? order_key(__ldg(l + e)) : 0u;
        id[i] = e;
    }
    // largest first; swapping only on a strict inequality keeps equal keys in
    // ascending id order
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
    int mine = -1;
    for (int k = 0; k < K; ++k) {
        const uint32_t m = __reduce_max_sync(0xffffffffu, key[0]);
        const uint32_t cand = key[0] == m ? (uint32_t)id[0] : 0xffffffffu;
        const uint32_t win = __reduce_min_sync(0xffffffffu, cand);
        if (lane == k) mine = (int)win;
        if (cand == win) {
#pragma unroll
            for (int i = 0; i + 1 < EPL; ++i) {
                key[i] = key[i + 1];
                id[i] = id[i + 1];
            }
            key[EPL - 1] = 0u;
        }
    }
    return mine;
}

template <int EPL> // experts per lane: E <= 32 * EPL
__global__ void __launch_bounds__(kRouterWarps * 32) k_router_topk(const float *__restrict__ logits, int T, int E,
                                                                    int K, int32_t *__restrict__ idx,
                                                                    float *__restrict__ w) {
    pdl_wait();
    pdl_launch_dependents();
    constexpr int B = id_bits(EPL);
    constexpr uint32_t M = (1u << B) - 1u;
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * kRouterWarps + (threadIdx.x >> 5);
    if (t >= T) return; // whole warp
    const float *l = logits + (int64_t)t * E;
    // one word per candidate: its key with the low B bits replaced by M - id,
    // so a larger word is a larger key, or an equal one with a lower id (a real
    // key is at least 2^23, so a real word is never 0, the empty candidate)
    uint32_t p[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        p[i] = e < E ? ((order_key(__ldcs(l + e)) & ~M) | (M - (uint32_t)e)) : 0u;
    }
#pragma unroll
    for (int r = 0; r < EPL; ++r) {
#pragma unroll
        for (int i = r & 1; i + 1 < EPL; i += 2) {
            const uint32_t hi = max(p[i], p[i + 1]), lo = min(p[i], p[i + 1]);
            p[i] = hi;
            p[i + 1] = lo;
        }
    }
    // K rounds of one reduction: the largest head word wins, and only the
    // lane holding it (words are distinct) pops its head
    uint32_t mine = 0u, last = 0u;
    for (int k = 0; k < K; ++k) {
        const uint32_t m = __reduce_max_sync(0xffffffffu, p[0]);
        if (lane == k) mine = m;
        if (p[0] == m) {
#pragma unroll
            for (int i = 0; i + 1 < EPL; ++i) p[i] = p[i + 1];
            p[EPL - 1] = 0u;
        }
        last = m;
    }
    // The words order candidates as the keys do, except two whose keys agree
    // above the low B bits. That can change the result only if two chosen
    // ones agree there, or an unchosen one agrees with the last chosen one
    // (every unchosen head is at most the last choice, so no deeper one can
    // agree without its lane's head agreeing too). Such warps redo the
    // selection with the full keys.
    const uint32_t next = __shfl_down_sync(0xffffffffu, mine, 1);
    const bool close = (lane + 1 < K && ((mine ^ next) & ~M) == 0u) || ((p[0] ^ last) & ~M) == 0u;
    int my_e;
    if (__any_sync(0xffffffffu, close))
        my_e = topk_exact<EPL>(l, lane, E, K);
    else
        my_e = lane < K ? (int)(M - (mine & M)) : -1;
    // weights from the chosen logits, read again (the words lost their low bits)
    const float v = lane < K ? __ldg(l + my_e) : 0.0f;
    const float vmax = __shfl_sync(0xffffffffu, v, 0);
    const float ex = lane < K ? expf(v - vmax) : 0.0f;
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
