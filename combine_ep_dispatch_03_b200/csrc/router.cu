// router.cu -- ep_router_topk: the gating step just before dispatch. For each
// token, the K experts with the largest logits and their router weights
// (softmax over the logits, renormalised over the K chosen experts).
//
// "Ultra-Large MoE Models: Open-Source Evolution and Heterogeneous Inference
// Adaptation", §2.1 (the gating network picks the top-K experts per token)
// and §3.1 (the top-K routing operator, a fused MoE-specific operator).
//
// Two kernels. For K <= 8 with E a multiple of 16, k_router_lanes (below)
// gives each token four lanes. Otherwise k_router_topk gives each token a warp:
// lane l holds experts l, l+32, ..., each as one 32-bit
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

// ---------------------------------------------------------------------------
// Four lanes per token (K <= 8, E a multiple of 16): eight tokens a warp.
// Lane s of a token reads its logits as 16-byte vectors (experts 16i + 4s ..
// 16i + 4s + 3), turns each into the packed word above, sorts them eight at a
// time with a 19-comparator network (Batcher's odd-even merge sort) and merges
// each sorted group into its running top eight (one bitonic merge step, then
// three half-cleaner stages). Two butterfly merges over the token's four lanes
// leave every lane with the token's top eight words. This needs no warp
// reduction and about a third of the instructions of one token per warp, which
// leaves the kernel bound by the logits' bytes. The largest word not kept is
// tracked through every merge, so the same two checks as above find the tokens
// whose packed words could have swapped two candidates; the whole warp redoes
// those with full keys.
// ---------------------------------------------------------------------------
constexpr int kLanesPerToken = 4;
constexpr int kLaneMaxK = 8; // the words a token's lanes keep

// the packed word of logit v of expert e (v + 0 turns -0 into +0, so equal
// logits get equal keys)
template <uint32_t M>
__device__ __forceinline__ uint32_t pack_word(float v, int e) {
    const uint32_t u = __float_as_uint(v + 0.0f);
    const uint32_t key = u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u);
    return (key & ~M) | (M - (uint32_t)e);
}

// compare-exchange: the larger word to a
__device__ __forceinline__ void cx(uint32_t &a, uint32_t &b) {
    const uint32_t hi = max(a, b);
    b = min(a, b);
    a = hi;
}

// sort eight words, largest first (Batcher's odd-even merge sort of 8)
__device__ __forceinline__ void sort8(uint32_t *w) {
    cx(w[0], w[1]); cx(w[2], w[3]); cx(w[4], w[5]); cx(w[6], w[7]);
    cx(w[0], w[2]); cx(w[1], w[3]); cx(w[4], w[6]); cx(w[5], w[7]);
    cx(w[1], w[2]); cx(w[5], w[6]);
    cx(w[0], w[4]); cx(w[1], w[5]); cx(w[2], w[6]); cx(w[3], w[7]);
    cx(w[2], w[4]); cx(w[3], w[5]);
    cx(w[1], w[2]); cx(w[3], w[4]); cx(w[5], w[6]);
}

// t := the eight largest of t and g (both sorted, largest first), sorted;
// rej := max(rej, the largest of the other eight)
__device__ __forceinline__ void merge8(uint32_t *t, const uint32_t *g, uint32_t &rej) {
    uint32_t lo = 0u;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t a = t[j], b = g[7 - j];
        t[j] = max(a, b); // largest first, then smallest, then larger again: bitonic
        lo = max(lo, min(a, b));
    }
    rej = max(rej, lo);
    cx(t[0], t[4]); cx(t[1], t[5]); cx(t[2], t[6]); cx(t[3], t[7]);
    cx(t[0], t[2]); cx(t[1], t[3]); cx(t[4], t[6]); cx(t[5], t[7]);
    cx(t[0], t[1]); cx(t[2], t[3]); cx(t[4], t[5]); cx(t[6], t[7]);
}

template <int EPL> // E <= 32 * EPL (sets the id bits and the exact path's shape)
__global__ void __launch_bounds__(kRouterWarps * 32) k_router_lanes(const float *__restrict__ logits, int T, int E,
                                                                     int K, int32_t *__restrict__ idx,
                                                                     float *__restrict__ w) {
    pdl_wait();
    pdl_launch_dependents();
    constexpr uint32_t M = (1u << id_bits(EPL)) - 1u;
    constexpr int kTok = 32 / kLanesPerToken; // tokens a warp
    __shared__ int s_fix[kRouterWarps][kLaneMaxK];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int s = lane & (kLanesPerToken - 1), tw = lane / kLanesPerToken;
    const int t0 = (blockIdx.x * kRouterWarps + wid) * kTok;
    if (t0 >= T) return; // whole warp
    const int t = t0 + tw;
    const bool live = t < T; // a lane past the last token works on token t0 and writes nothing
    const float *l = logits + (int64_t)(live ? t : t0) * E;
    const float4 *row = reinterpret_cast<const float4 *>(l);
    const int nv = E >> 4; // 16-byte vectors a lane reads
    // Two groups of eight words an iteration: the sort of the second group
    // is independent of the first group's merge, so the two overlap.
    uint32_t top[8], rej = 0u;
    float4 v4[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v4[u] = u < nv ? __ldcs(row + 4 * u + s) : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i0 = 0; i0 < nv; i0 += 4) {
        float4 nx[4]; // the next iteration's vectors go out before this one's sorts
#pragma unroll
        for (int u = 0; u < 4; ++u)
            nx[u] = i0 + 4 + u < nv ? __ldcs(row + 4 * (i0 + 4 + u) + s) : make_float4(0.f, 0.f, 0.f, 0.f);
        uint32_t g[2][8];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = 16 * (i0 + u) + 4 * s;
            const bool has = i0 + u < nv;
            uint32_t *gw = g[u >> 1] + 4 * (u & 1);
            gw[0] = has ? pack_word<M>(v4[u].x, e) : 0u;
            gw[1] = has ? pack_word<M>(v4[u].y, e + 1) : 0u;
            gw[2] = has ? pack_word<M>(v4[u].z, e + 2) : 0u;
            gw[3] = has ? pack_word<M>(v4[u].w, e + 3) : 0u;
        }
        sort8(g[0]);
        sort8(g[1]);
        if (i0 == 0) {
#pragma unroll
            for (int j = 0; j < 8; ++j) top[j] = g[0][j];
        } else {
            merge8(top, g[0], rej);
        }
        merge8(top, g[1], rej);
#pragma unroll
        for (int u = 0; u < 4; ++u) v4[u] = nx[u];
    }
    // the token's four lanes merge their lists (every lane ends with all of it)
#pragma unroll
    for (int d = 1; d < kLanesPerToken; d <<= 1) {
        uint32_t o[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) o[j] = __shfl_xor_sync(0xffffffffu, top[j], d);
        rej = max(rej, __shfl_xor_sync(0xffffffffu, rej, d));
        merge8(top, o, rej);
    }
    // the two checks on the packed words: two chosen words, or the last chosen
    // and the best unchosen one, that agree above the low bits
    uint32_t last = top[0], unchosen = rej;
    bool close = false;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        if (j + 1 < K && j + 1 < 8) close |= ((top[j] ^ top[j + 1]) & ~M) == 0u;
        if (j == K - 1) last = top[j];
        if (j == K) unchosen = top[j];
    }
    close |= ((last ^ unchosen) & ~M) == 0u;
    // this lane's choices k = s and s + 4
    int my_e[2] = {-1, -1};
#pragma unroll
    for (int jj = 0; jj < 2; ++jj) {
        uint32_t wd = 0u;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (j == s + 4 * jj) wd = top[j];
        if (s + 4 * jj < K) my_e[jj] = (int)(M - (wd & M));
    }
    unsigned redo = __ballot_sync(0xffffffffu, live && close && s == 0);
    while (redo) { // warp-uniform: the whole warp redoes one token with full keys
        const int src = (__ffs(redo) - 1) / kLanesPerToken;
        redo &= redo - 1;
        const int id = topk_exact<EPL>(logits + (int64_t)(t0 + src) * E, lane, E, K);
        if (lane < K) s_fix[wid][lane] = id;
        __syncwarp();
        if (tw == src)
#pragma unroll
            for (int jj = 0; jj < 2; ++jj)
                if (s + 4 * jj < K) my_e[jj] = s_fix[wid][s + 4 * jj];
        __syncwarp();
    }
    // weights from the chosen logits (read again: the words lost their low bits)
    float ex[2];
    float v[2];
#pragma unroll
    for (int jj = 0; jj < 2; ++jj) v[jj] = s + 4 * jj < K ? __ldg(l + my_e[jj]) : 0.0f;
    const int base = lane & ~(kLanesPerToken - 1);
    const float vmax = __shfl_sync(0xffffffffu, v[0], base); // choice 0: slot 0 of lane s = 0
#pragma unroll
    for (int jj = 0; jj < 2; ++jj) ex[jj] = s + 4 * jj < K ? expf(v[jj] - vmax) : 0.0f;
    float sum = 0.0f;
#pragma unroll
    for (int k = 0; k < kLaneMaxK; ++k) {
        const float e = __shfl_sync(0xffffffffu, ex[k >> 2], base | (k & 3));
        if (k < K) sum = __fadd_rn(sum, e); // fixed k order
    }
    if (live)
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            const int k = s + 4 * jj;
            if (k < K) {
                idx[(int64_t)t * K + k] = my_e[jj];
                w[(int64_t)t * K + k] = __fdiv_rn(ex[jj], sum);
            }
        }
}

template <int EPL>
cudaError_t launch_router(const float *logits, int T, int E, int K, int32_t *idx, float *w, cudaStream_t st) {
    const bool lanes = K <= kLaneMaxK && E % 16 == 0 && ((uintptr_t)logits & 15) == 0;
    if (lanes) {
        const int per_cta = kRouterWarps * 32 / kLanesPerToken;
        return launch_pdl(k_router_lanes<EPL>, dim3((T + per_cta - 1) / per_cta), dim3(kRouterWarps * 32), 0, st,
                          logits, T, E, K, idx, w);
    }
    return launch_pdl(k_router_topk<EPL>, dim3((T + kRouterWarps - 1) / kRouterWarps), dim3(kRouterWarps * 32), 0,
                      st, logits, T, E, K, idx, w);
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
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t err;
    const int epl = (E + 31) / 32;
    if (epl <= 1)
        err = launch_router<1>(logits, T, E, K, topk_idx, topk_w, st);
    else if (epl <= 2)
        err = launch_router<2>(logits, T, E, K, topk_idx, topk_w, st);
    else if (epl <= 4)
        err = launch_router<4>(logits, T, E, K, topk_idx, topk_w, st);
    else if (epl <= 8)
        err = launch_router<8>(logits, T, E, K, topk_idx, topk_w, st);
    else if (epl <= 16)
        err = launch_router<16>(logits, T, E, K, topk_idx, topk_w, st);
    else
        err = launch_router<32>(logits, T, E, K, topk_idx, topk_w, st);
    return err == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}
