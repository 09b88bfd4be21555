// world.cu -- expert parallelism across GPUs, one rank per GPU: the send and
// receive halves of dispatch over peer memory, completion flags, combine that
// reads the peers' expert outputs, and CUDA IPC for building the peer table.
//
// NCCL EP paper (arXiv 2603.13606): the staged mode splits dispatch and
// combine into send and receive phases (Table II, Fig. 2); LL mode runs as an
// all-to-all mesh and combine reduces per token at the receiver (Table III).
// MoonEP article, para. 4: rows go straight into expert-grouped positions on
// the remote rank, with no staging copy through a communication buffer.
//
// The routing of a world plan (global rows) is in route.cu. Here a global row
// g is mapped to its rank r (the last r with rank_off[r] <= g) and local row
// g - rank_off[r], and every row moves with plain 16-byte stores (dispatch)
// or loads (combine) through the peer table: over NVLink when the table holds
// other GPUs' mapped buffers, within one HBM when it holds local ones. No bulk
// copy engine or cluster-wide broadcast load touches a peer's memory.
#include <string.h>

#include "bulk.cuh"
#include "ep_internal.cuh"
#include "rows.cuh"

namespace epb {
namespace {

// the peers' receive arrays, passed by value as a kernel parameter
struct PeerRows {
    uint8_t *x[EP_MAX_PEERS];
    float *scales[EP_MAX_PEERS];
    float *w[EP_MAX_PEERS];
    int32_t *expert[EP_MAX_PEERS];
    int64_t cap; // rows of every rank's receive buffer
};

struct PeerFlags {
    uint32_t *f[EP_MAX_PEERS];
};

// The rank holding global row g: the last r with roff[r] <= g (roff ascending
// from roff[0] = 0; empty ranks share their offset with the next rank).
__device__ __forceinline__ int row_rank(const int32_t *roff, int R, int g) {
    int lo = 0, hi = R - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (roff[mid] <= g)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

// Threads k < K of the CTA: rank and local row of pair (t, k), or rank -1 for
// a pair without a row or with a row beyond the capacity (flagged).
__device__ __forceinline__ void stage_peer_rows(const int32_t *__restrict__ dest_row,
                                                const int32_t *__restrict__ rank_off, int R, int K, int64_t pb,
                                                int64_t cap, int32_t *s_roff, int *s_rank, int64_t *s_lrow,
                                                uint32_t *status) {
    for (int i = threadIdx.x; i <= R; i += blockDim.x) s_roff[i] = rank_off[i];
    __syncthreads();
    if (threadIdx.x < K) {
        const int g = dest_row[pb + threadIdx.x];
        int r = -1;
        int64_t lr = -1;
        if (g >= 0) {
            r = row_rank(s_roff, R, g);
            lr = g - s_roff[r];
            if (lr >= cap) {
                if (status) atomicOr(status, EP_FLAG_CAPACITY);
                r = -1;
            }
        }
        s_rank[threadIdx.x] = r;
        s_lrow[threadIdx.x] = lr;
    }
}

// dispatch send, bf16 rows: one CTA per (token, row part), VPT 16-byte vectors
// a thread; the token's vectors are read once and stored K times. SCALE (the
// combine backward across ranks): each row is bf16(w[t,k] * x[t]) instead,
// one fp32 product and one rounding, and no weights or ids are recorded.
template <int VPT, bool SCALE>
__global__ void __launch_bounds__(256) k_dispatch_peers(const uint4 *__restrict__ x, const int32_t *__restrict__ idx,
                                                        const float *__restrict__ w,
                                                        const int32_t *__restrict__ dest_row,
                                                        const int32_t *__restrict__ rank_off, int R, int K, int nvec,
                                                        int part, PeerRows pr, uint32_t *__restrict__ status) {
    __shared__ int32_t s_roff[EP_MAX_PEERS + 1];
    __shared__ int s_rank[kMaxTopk];
    __shared__ int64_t s_lrow[kMaxTopk];
    __shared__ uint4 *s_dst[kMaxTopk];
    __shared__ float s_wk[kMaxTopk];
    const int t = blockIdx.x;
    const int64_t pb = (int64_t)t * K;
    const int cb = blockIdx.y * part, n = min(part, nvec - cb);
    const uint4 *src = x + (int64_t)t * nvec + cb;
    const int step = VPT * blockDim.x;
    uint4 v[VPT];
    load_slab<VPT>(src, 0, n, v); // before the wait: the routing never writes x
    pdl_wait();
    stage_peer_rows(dest_row, rank_off, R, K, pb, pr.cap, s_roff, s_rank, s_lrow,
                    blockIdx.y == 0 ? status : nullptr);
    if (threadIdx.x < K) {
        const int r = s_rank[threadIdx.x];
        const int64_t lr = s_lrow[threadIdx.x];
        s_dst[threadIdx.x] = r >= 0 ? reinterpret_cast<uint4 *>(pr.x[r]) + lr * nvec + cb : nullptr;
        if (SCALE) {
            s_wk[threadIdx.x] = w[pb + threadIdx.x];
        } else if (r >= 0 && blockIdx.y == 0) {
            if (pr.w[r]) pr.w[r][lr] = w[pb + threadIdx.x];
            if (pr.expert[r]) pr.expert[r][lr] = idx[pb + threadIdx.x];
        }
    }
    __syncthreads();
    for (int c0 = 0; c0 < n; c0 += step) {
        if (c0 > 0) load_slab<VPT>(src, c0, n, v);
        for (int k = 0; k < K; ++k) {
            uint4 *dst = s_dst[k];
            if (!dst) continue;
            const float wk = SCALE ? s_wk[k] : 1.0f;
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int c = c0 + threadIdx.x + i * blockDim.x;
                if (c >= n) continue;
                if (SCALE) {
                    float f[8];
                    unpack8(v[i], f);
#pragma unroll
                    for (int u = 0; u < 8; ++u) f[u] = __fmul_rn(wk, f[u]);
                    dst[c] = pack8(f);
                } else {
                    dst[c] = v[i];
                }
            }
        }
    }
}

// dispatch send, FP8 rows: the same cast as the single-GPU FP8 dispatch (one
// thread per 16-element chunk, the 8 lanes of a 128-element block reduce its
// amax), then the codes and scales stored to each pair's rank.
template <int CPT>
__global__ void __launch_bounds__(256) k_dispatch_peers_fp8(const uint4 *__restrict__ x,
                                                            const int32_t *__restrict__ idx,
                                                            const float *__restrict__ w,
                                                            const int32_t *__restrict__ dest_row,
                                                            const int32_t *__restrict__ rank_off, int R, int K,
                                                            int nchunk, int part, PeerRows pr,
                                                            uint32_t *__restrict__ status) {
    __shared__ int32_t s_roff[EP_MAX_PEERS + 1];
    __shared__ int s_rank[kMaxTopk];
    __shared__ int64_t s_lrow[kMaxTopk];
    __shared__ uint4 *s_dst[kMaxTopk];
    __shared__ float *s_sc[kMaxTopk];
    const int t = blockIdx.x;
    const int64_t pb = (int64_t)t * K;
    const int nb = nchunk >> 3; // 128-element blocks per row
    const int cb = blockIdx.y * part, n = min(part, nchunk - cb); // part: whole blocks
    const uint4 *src = x + (int64_t)t * 2 * nchunk + 2 * cb;
    const int step = CPT * blockDim.x;
    uint4 a[CPT], b[CPT];
    load_pairs<CPT>(src, 0, n, a, b); // before the wait: the routing never writes x
    pdl_wait();
    stage_peer_rows(dest_row, rank_off, R, K, pb, pr.cap, s_roff, s_rank, s_lrow,
                    blockIdx.y == 0 ? status : nullptr);
    if (threadIdx.x < K) {
        const int r = s_rank[threadIdx.x];
        const int64_t lr = s_lrow[threadIdx.x];
        s_dst[threadIdx.x] = r >= 0 ? reinterpret_cast<uint4 *>(pr.x[r]) + lr * nchunk + cb : nullptr;
        s_sc[threadIdx.x] = r >= 0 ? pr.scales[r] + lr * nb + (cb >> 3) : nullptr;
        if (r >= 0 && blockIdx.y == 0) {
            if (pr.w[r]) pr.w[r][lr] = w[pb + threadIdx.x];
            if (pr.expert[r]) pr.expert[r][lr] = idx[pb + threadIdx.x];
        }
    }
    __syncthreads();
    for (int c0 = 0; c0 < n; c0 += step) {
        if (c0 > 0) load_pairs<CPT>(src, c0, n, a, b);
        uint4 q[CPT];
        float sc[CPT];
#pragma unroll
        for (int i = 0; i < CPT; ++i) quant_chunk(a[i], b[i], q[i], sc[i]);
        for (int k = 0; k < K; ++k) {
            uint4 *dst = s_dst[k];
            if (!dst) continue;
            float *scr = s_sc[k];
#pragma unroll
            for (int i = 0; i < CPT; ++i) {
                const int c = c0 + threadIdx.x + i * blockDim.x;
                if (c < n) {
                    dst[c] = q[i];
                    if ((c & 7) == 0) scr[c >> 3] = sc[i];
                }
            }
        }
    }
}

// combine across ranks: out[t] = bf16(fold_k fmaf(w[t,k], y_k, acc)) with y_k
// the pair's row in its rank's expert outputs, k in order, acc from +0. UNIT
// (the dispatch backward across ranks): an unweighted fp32 sum in k order.
template <int CPT, bool UNIT>
__global__ void __launch_bounds__(256) k_combine_peers(PeerRows pr, const float *__restrict__ w,
                                                       const int32_t *__restrict__ dest_row,
                                                       const int32_t *__restrict__ rank_off, int R, int K, int nvec,
                                                       int part, uint4 *__restrict__ out) {
    __shared__ int32_t s_roff[EP_MAX_PEERS + 1];
    __shared__ int s_rank[kMaxTopk];
    __shared__ int64_t s_lrow[kMaxTopk];
    __shared__ const uint4 *s_src[kMaxTopk];
    __shared__ float s_w[kMaxTopk];
    pdl_wait();
    const int t = blockIdx.x;
    const int64_t pb = (int64_t)t * K;
    const int cb = blockIdx.y * part, n = min(part, nvec - cb);
    stage_peer_rows(dest_row, rank_off, R, K, pb, pr.cap, s_roff, s_rank, s_lrow, nullptr);
    if (threadIdx.x < K) {
        const int r = s_rank[threadIdx.x];
        s_src[threadIdx.x] =
            r >= 0 ? reinterpret_cast<const uint4 *>(pr.x[r]) + s_lrow[threadIdx.x] * nvec + cb : nullptr;
        s_w[threadIdx.x] = UNIT ? 1.0f : w[pb + threadIdx.x];
    }
    __syncthreads();
    const int step = CPT * blockDim.x;
    for (int c0 = 0; c0 < n; c0 += step) {
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            const int c = c0 + threadIdx.x + i * blockDim.x;
            if (c >= n) continue;
            float acc[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) acc[u] = 0.0f;
            for (int k0 = 0; k0 < K; k0 += 8) {
                uint4 v[8];
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const int k = k0 + kk;
                    const uint4 *p = k < K ? s_src[k] : nullptr;
                    v[kk] = p ? p[c] : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const int k = k0 + kk;
                    if (k >= K || !s_src[k]) continue;
                    float f[8];
                    unpack8(v[kk], f);
                    if (UNIT) {
#pragma unroll
                        for (int u = 0; u < 8; ++u) acc[u] = __fadd_rn(acc[u], f[u]);
                    } else {
                        const float wk = s_w[k];
#pragma unroll
                        for (int u = 0; u < 8; ++u) acc[u] = __fmaf_rn(wk, f[u], acc[u]);
                    }
                }
            }
            out[(int64_t)t * nvec + cb + c] = pack8(acc);
        }
    }
}

// replica-gradient reduce across ranks: this rank (own experts [e0, e0 + g))
// adds, for each of its experts with replicas, the replica slots' gradients in
// ascending slot order (each read from the slot's rank through the table) to
// its own owner rows (fp32, in place). A persistent grid over (replicated
// expert, 4096-element chunk) items; experts of other ranks are skipped.
struct PeerGrads {
    const float4 *rep[EP_MAX_PEERS]; // rank r's replica gradients [S, G] fp32
};

constexpr int kRedPeerThreads = 256, kRedPeerUnroll = 4;

__global__ void __launch_bounds__(kRedPeerThreads) k_reduce_peers(PeerGrads pg, float4 *__restrict__ owner,
                                                                  const int32_t *__restrict__ red_experts,
                                                                  const int32_t *__restrict__ red_count,
                                                                  const int32_t *__restrict__ red_list,
                                                                  const int32_t *__restrict__ red_n, int R, int S,
                                                                  int e0, int g, int64_t G4) {
    pdl_wait();
    const int nred = *red_count;
    const int64_t chunk = (int64_t)kRedPeerThreads * kRedPeerUnroll;
    const int per = (int)((G4 + chunk - 1) / chunk); // chunks per expert (host-checked to fit)
    const int items = nred * per;
    for (int it = blockIdx.x; it < items; it += gridDim.x) {
        const int e = red_experts[it / per];
        if (e < e0 || e >= e0 + g) continue; // another rank's expert
        const int64_t base = (int64_t)(it % per) * chunk + threadIdx.x;
        const int n = red_n[e];
        const int32_t *lst = red_list + (int64_t)e * R;
        float4 *o = owner + (int64_t)(e - e0) * G4;
        float4 acc[kRedPeerUnroll];
#pragma unroll
        for (int u = 0; u < kRedPeerUnroll; ++u) {
            const int64_t i = base + (int64_t)u * kRedPeerThreads;
            acc[u] = i < G4 ? o[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        for (int a = 0; a < n; ++a) {
            const int key = lst[a]; // r * S + s
            const float4 *src = pg.rep[key / S] + (int64_t)(key % S) * G4;
#pragma unroll
            for (int u = 0; u < kRedPeerUnroll; ++u) {
                const int64_t i = base + (int64_t)u * kRedPeerThreads;
                if (i < G4) {
                    const float4 v = src[i];
                    acc[u].x = __fadd_rn(acc[u].x, v.x);
                    acc[u].y = __fadd_rn(acc[u].y, v.y);
                    acc[u].z = __fadd_rn(acc[u].z, v.z);
                    acc[u].w = __fadd_rn(acc[u].w, v.w);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kRedPeerUnroll; ++u) {
            const int64_t i = base + (int64_t)u * kRedPeerThreads;
            if (i < G4) o[i] = acc[u];
        }
    }
}

// replica weight prefetch across ranks: for each replica slot s of this rank
// that the world plan fills with expert e, copy e's weights from its owner's
// table entry (e's row among the owner's experts). A persistent grid over
// (slot, 16 KB chunk) items; empty slots are skipped.
constexpr int kCopyPeerThreads = 256, kCopyPeerUnroll = 4;

__global__ void __launch_bounds__(kCopyPeerThreads) k_prefetch_peers(PeerRows pw, uint4 *__restrict__ slots,
                                                                     const int32_t *__restrict__ replica_expert,
                                                                     int rank, int S, int g, int64_t V) {
    pdl_wait();
    const int64_t chunk = (int64_t)kCopyPeerThreads * kCopyPeerUnroll;
    const int per = (int)((V + chunk - 1) / chunk); // chunks per expert (host-checked to fit)
    const int items = S * per;
    for (int it = blockIdx.x; it < items; it += gridDim.x) {
        const int s = it / per;
        const int e = replica_expert[rank * S + s];
        if (e < 0) continue; // an empty slot
        const int o = e / g;
        const uint4 *src = reinterpret_cast<const uint4 *>(pw.x[o]) + (int64_t)(e - o * g) * V;
        uint4 *dst = slots + (int64_t)s * V;
        const int64_t base = (int64_t)(it % per) * chunk + threadIdx.x;
        uint4 v[kCopyPeerUnroll];
#pragma unroll
        for (int u = 0; u < kCopyPeerUnroll; ++u) {
            const int64_t i = base + (int64_t)u * kCopyPeerThreads;
            if (i < V) v[u] = src[i];
        }
#pragma unroll
        for (int u = 0; u < kCopyPeerUnroll; ++u) {
            const int64_t i = base + (int64_t)u * kCopyPeerThreads;
            if (i < V) dst[i] = v[u];
        }
    }
}

__device__ __forceinline__ void st_release_sys(uint32_t *p, uint32_t v) {
    asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// signal: after the kernels before it (griddepcontrol.wait), a system-scope
// fence, then flags[r][rank] = epoch on every rank r (release).
__global__ void __launch_bounds__(64) k_signal(PeerFlags pf, int R, int rank, uint32_t epoch) {
    pdl_wait();
    __threadfence_system();
    for (int r = threadIdx.x; r < R; r += blockDim.x) st_release_sys(pf.f[r] + rank, epoch);
}

// wait: thread s polls flags[s] (acquire) until it reaches epoch (wrapping
// 32-bit comparison), for at most limit_ns; a thread that gives up sets
// EP_FLAG_WAIT_TIMEOUT. Nothing else runs in this kernel, and the kernels
// after it start only when it has completed.
__global__ void __launch_bounds__(64) k_wait(const uint32_t *flags, int R, uint32_t epoch, uint64_t limit_ns,
                                             uint32_t *status) {
    pdl_wait();
    for (int s = threadIdx.x; s < R; s += blockDim.x) {
        const uint64_t t0 = global_ns();
        while ((int32_t)(ld_acquire_sys(flags + s) - epoch) < 0) {
            if (global_ns() - t0 > limit_ns) {
                atomicOr(status, EP_FLAG_WAIT_TIMEOUT);
                break;
            }
            __nanosleep(256);
        }
    }
}

} // namespace
} // namespace epb

using namespace epb;

static inline bool aligned_to(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

// common checks of a peer table against a handle
static ep_status_t check_table(const ep_handle_t *h, const ep_peer_table_t *pt, bool need_x) {
    if (!pt || pt->num_ranks != h->d.R || h->d.R > EP_MAX_PEERS || pt->capacity_rows < 0) return EP_ERR_INVALID_ARG;
    if (pt->capacity_rows > INT32_MAX) return EP_ERR_INVALID_ARG;
    if (need_x)
        for (int r = 0; r < h->d.R; ++r)
            if (!pt->recv_x[r] || !aligned_to(pt->recv_x[r], 16)) return EP_ERR_INVALID_ARG;
    return EP_OK;
}

static void fill_rows(const ep_peer_table_t *pt, int R, PeerRows *pr) {
    memset(pr, 0, sizeof *pr);
    for (int r = 0; r < R; ++r) {
        pr->x[r] = (uint8_t *)pt->recv_x[r];
        pr->scales[r] = pt->recv_scales[r];
        pr->w[r] = pt->recv_w[r];
        pr->expert[r] = pt->recv_expert[r];
    }
    pr->cap = pt->capacity_rows;
}

extern "C" {

ep_status_t ep_world_recv_rows(const ep_config_t *cfg, int64_t *rows) {
    Dims d;
    if (!rows) return EP_ERR_INVALID_ARG;
    const ep_status_t s = derive_dims(cfg, &d);
    if (s != EP_OK) return s;
    if (d.mode == EP_MODE_LL)
        *rows = (int64_t)d.g * d.cap;
    else
        *rows = d.balanced ? d.L : (int64_t)d.R * d.L; // ceil(R*L / R) = L with a plan
    return EP_OK;
}

ep_status_t ep_plan_local_counts(ep_handle_t *h, const int32_t *topk_idx, int32_t *counts, void *stream) {
    if (!h || !counts || !aligned_to(counts, 4)) return EP_ERR_INVALID_ARG;
    if (h->d.T > 0 && (!topk_idx || !aligned_to(topk_idx, 4))) return EP_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    h->planned = 0;
    h->counts_ready = 0;
    if (launch_plan_local_counts(h->d, h->ws, topk_idx, st) != cudaSuccess) return EP_ERR_CUDA;
    if (cudaMemcpyAsync(counts, h->ws.cnt, sizeof(int32_t) * h->d.E, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return EP_ERR_CUDA;
    h->counts_ready = 1;
    return EP_OK;
}

ep_status_t ep_plan_world(ep_handle_t *h, const int32_t *world_counts, int32_t rank, void *stream) {
    if (!h || !world_counts || !aligned_to(world_counts, 4) || rank < 0 || rank >= h->d.R) return EP_ERR_INVALID_ARG;
    if (!h->counts_ready) return EP_ERR_NOT_PLANNED;
    if (h->d.R > EP_MAX_PEERS) return EP_ERR_UNSUPPORTED;
    if ((int64_t)h->d.R * h->d.L > INT32_MAX / 2) return EP_ERR_INVALID_ARG; // global rows fit 31 bits
    Dims dw = h->d;
    dw.world = 1;
    if (route_smem_world(dw) > (size_t)kMaxRouteSmem || route_smem_assign(dw) > (size_t)kMaxRouteSmem)
        return EP_ERR_UNSUPPORTED;
    if (launch_plan_world(h->d, h->ws, world_counts, rank, (cudaStream_t)stream) != cudaSuccess) return EP_ERR_CUDA;
    h->planned = 2;
    h->world_rank = rank;
    return EP_OK;
}

ep_status_t ep_dispatch_peers(ep_handle_t *h, const void *x, const int32_t *topk_idx, const float *topk_w,
                              const ep_peer_table_t *peers, void *stream) {
    if (!h) return EP_ERR_INVALID_ARG;
    if (h->planned != 2) return h->planned == 1 ? EP_ERR_UNSUPPORTED : EP_ERR_NOT_PLANNED;
    const Dims &d = h->d;
    ep_status_t s = check_table(h, peers, true);
    if (s != EP_OK) return s;
    bool any_w = false, any_e = false;
    for (int r = 0; r < d.R; ++r) {
        if (peers->recv_w[r] && !aligned_to(peers->recv_w[r], 4)) return EP_ERR_INVALID_ARG;
        if (peers->recv_expert[r] && !aligned_to(peers->recv_expert[r], 4)) return EP_ERR_INVALID_ARG;
        if (d.fp8 && (!peers->recv_scales[r] || !aligned_to(peers->recv_scales[r], 4))) return EP_ERR_INVALID_ARG;
        if (!d.fp8 && peers->recv_scales[r]) return EP_ERR_INVALID_ARG;
        any_w |= peers->recv_w[r] != nullptr;
        any_e |= peers->recv_expert[r] != nullptr;
    }
    if (d.T == 0) return EP_OK;
    if (!x || !aligned_to(x, 16)) return EP_ERR_INVALID_ARG;
    if (any_w && (!topk_w || !aligned_to(topk_w, 4))) return EP_ERR_INVALID_ARG;
    if (any_e && (!topk_idx || !aligned_to(topk_idx, 4))) return EP_ERR_INVALID_ARG;
    PeerRows pr;
    fill_rows(peers, d.R, &pr);
    cudaStream_t st = (cudaStream_t)stream;
    int per, threads;
    cudaError_t err;
    if (d.fp8) {
        const int nchunk = d.H / 16;
        const int part = row_part(d.T, nchunk);
        const dim3 grid(d.T, (nchunk + part - 1) / part);
        pick_shape(part, &per, &threads);
#define EPB_PEER_FP8(C)                                                                                              \
    launch_pdl(k_dispatch_peers_fp8<C>, grid, dim3(threads), 0, st, (const uint4 *)x, topk_idx, topk_w, h->ws.dest_row, \
               h->ws.rank_off, d.R, d.K, nchunk, part, pr, h->ws.flags)
        err = per == 1 ? EPB_PEER_FP8(1) : per == 2 ? EPB_PEER_FP8(2) : per == 4 ? EPB_PEER_FP8(4) : EPB_PEER_FP8(8);
#undef EPB_PEER_FP8
    } else {
        const int nvec = d.H / 8;
        const int part = row_part(d.T, nvec);
        const dim3 grid(d.T, (nvec + part - 1) / part);
        pick_shape(part, &per, &threads);
#define EPB_PEER_BF16(V)                                                                                             \
    launch_pdl(k_dispatch_peers<V, false>, grid, dim3(threads), 0, st, (const uint4 *)x, topk_idx, topk_w,             \
               h->ws.dest_row, h->ws.rank_off, d.R, d.K, nvec, part, pr, h->ws.flags)
        err = per == 1 ? EPB_PEER_BF16(1) : per == 2 ? EPB_PEER_BF16(2) : per == 4 ? EPB_PEER_BF16(4) : EPB_PEER_BF16(8);
#undef EPB_PEER_BF16
    }
    return err == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

ep_status_t ep_signal_peers(ep_handle_t *h, const ep_peer_table_t *peers, uint32_t epoch, void *stream) {
    if (!h) return EP_ERR_INVALID_ARG;
    ep_status_t s = check_table(h, peers, false);
    if (s != EP_OK) return s;
    PeerFlags pf;
    memset(&pf, 0, sizeof pf);
    for (int r = 0; r < h->d.R; ++r) {
        if (!peers->flags[r] || !aligned_to(peers->flags[r], 4)) return EP_ERR_INVALID_ARG;
        pf.f[r] = peers->flags[r];
    }
    // the rank index of this handle: the one ep_plan_world was given
    if (h->planned != 2) return EP_ERR_NOT_PLANNED;
    const cudaError_t err =
        launch_pdl(k_signal, dim3(1), dim3(64), 0, (cudaStream_t)stream, pf, h->d.R, h->world_rank, epoch);
    return err == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

ep_status_t ep_wait_peers(ep_handle_t *h, const uint32_t *flags, uint32_t epoch, int64_t timeout_us, void *stream) {
    if (!h || !flags || !aligned_to(flags, 4) || timeout_us < 0 || timeout_us > 600000000) return EP_ERR_INVALID_ARG;
    const uint64_t limit_ns = timeout_us == 0 ? kWaitLimitNs : (uint64_t)timeout_us * 1000ull;
    const cudaError_t err =
        launch_pdl(k_wait, dim3(1), dim3(64), 0, (cudaStream_t)stream, flags, h->d.R, epoch, limit_ns, h->ws.flags);
    return err == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

ep_status_t ep_combine_peers(ep_handle_t *h, const ep_peer_table_t *peers, const float *topk_w, void *out,
                             void *stream) {
    if (!h) return EP_ERR_INVALID_ARG;
    if (h->planned != 2) return h->planned == 1 ? EP_ERR_UNSUPPORTED : EP_ERR_NOT_PLANNED;
    const Dims &d = h->d;
    ep_status_t s = check_table(h, peers, true);
    if (s != EP_OK) return s;
    if (d.T == 0) return EP_OK;
    if (!topk_w || !out || !aligned_to(topk_w, 4) || !aligned_to(out, 16)) return EP_ERR_INVALID_ARG;
    PeerRows pr;
    fill_rows(peers, d.R, &pr);
    const int nvec = d.H / 8;
    const int part = row_part(d.T, nvec);
    const dim3 grid(d.T, (nvec + part - 1) / part);
    int per, threads;
    pick_shape(part, &per, &threads);
    cudaStream_t st = (cudaStream_t)stream;
#define EPB_PEER_COMB(C)                                                                                             \
    launch_pdl(k_combine_peers<C, false>, grid, dim3(threads), 0, st, pr, topk_w, h->ws.dest_row, h->ws.rank_off, d.R, \
               d.K, nvec, part, (uint4 *)out)
    const cudaError_t err =
        per == 1 ? EPB_PEER_COMB(1) : per == 2 ? EPB_PEER_COMB(2) : per == 4 ? EPB_PEER_COMB(4) : EPB_PEER_COMB(8);
#undef EPB_PEER_COMB
    return err == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

ep_status_t ep_combine_backward_peers(ep_handle_t *h, const void *grad_out, const float *topk_w,
                                      const ep_peer_table_t *grad_rows, void *stream) {
    if (!h) return EP_ERR_INVALID_ARG;
    if (h->planned != 2) return h->planned == 1 ? EP_ERR_UNSUPPORTED : EP_ERR_NOT_PLANNED;
    const Dims &d = h->d;
    ep_status_t s = check_table(h, grad_rows, true);
    if (s != EP_OK) return s;
    if (d.T == 0) return EP_OK;
    if (!grad_out || !topk_w || !aligned_to(grad_out, 16) || !aligned_to(topk_w, 4)) return EP_ERR_INVALID_ARG;
    PeerRows pr;
    fill_rows(grad_rows, d.R, &pr);
    for (int r = 0; r < d.R; ++r) { // gradient rows only: no weights, ids or scales recorded
        pr.scales[r] = nullptr;
        pr.w[r] = nullptr;
        pr.expert[r] = nullptr;
    }
    const int nvec = d.H / 8;
    const int part = row_part(d.T, nvec);
    const dim3 grid(d.T, (nvec + part - 1) / part);
    int per, threads;
    pick_shape(part, &per, &threads);
    cudaStream_t st = (cudaStream_t)stream;
#define EPB_PEER_CBWD(V)                                                                                             \
    launch_pdl(k_dispatch_peers<V, true>, grid, dim3(threads), 0, st, (const uint4 *)grad_out, (const int32_t *)nullptr,\
               topk_w, h->ws.dest_row, h->ws.rank_off, d.R, d.K, nvec, part, pr, h->ws.flags)
    const cudaError_t err =
        per == 1 ? EPB_PEER_CBWD(1) : per == 2 ? EPB_PEER_CBWD(2) : per == 4 ? EPB_PEER_CBWD(4) : EPB_PEER_CBWD(8);
#undef EPB_PEER_CBWD
    return err == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

ep_status_t ep_dispatch_backward_peers(ep_handle_t *h, const ep_peer_table_t *grad_rows, void *grad_x,
                                       void *stream) {
    if (!h) return EP_ERR_INVALID_ARG;
    if (h->planned != 2) return h->planned == 1 ? EP_ERR_UNSUPPORTED : EP_ERR_NOT_PLANNED;
    const Dims &d = h->d;
    ep_status_t s = check_table(h, grad_rows, true);
    if (s != EP_OK) return s;
    if (d.T == 0) return EP_OK;
    if (!grad_x || !aligned_to(grad_x, 16)) return EP_ERR_INVALID_ARG;
    PeerRows pr;
    fill_rows(grad_rows, d.R, &pr);
    const int nvec = d.H / 8;
    const int part = row_part(d.T, nvec);
    const dim3 grid(d.T, (nvec + part - 1) / part);
    int per, threads;
    pick_shape(part, &per, &threads);
    cudaStream_t st = (cudaStream_t)stream;
#define EPB_PEER_DBWD(C)                                                                                             \
    launch_pdl(k_combine_peers<C, true>, grid, dim3(threads), 0, st, pr, (const float *)nullptr, h->ws.dest_row,      \
               h->ws.rank_off, d.R, d.K, nvec, part, (uint4 *)grad_x)
    const cudaError_t err =
        per == 1 ? EPB_PEER_DBWD(1) : per == 2 ? EPB_PEER_DBWD(2) : per == 4 ? EPB_PEER_DBWD(4) : EPB_PEER_DBWD(8);
#undef EPB_PEER_DBWD
    return err == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

ep_status_t ep_reduce_replica_grads_peers(ep_handle_t *h, const ep_peer_table_t *replica_grads, float *owner_grad,
                                          void *stream) {
    if (!h) return EP_ERR_INVALID_ARG;
    if (!h->d.balanced) return EP_ERR_UNSUPPORTED;
    if (h->planned != 2) return h->planned == 1 ? EP_ERR_UNSUPPORTED : EP_ERR_NOT_PLANNED;
    const Dims &d = h->d;
    if (!replica_grads || replica_grads->num_ranks != d.R || d.R > EP_MAX_PEERS) return EP_ERR_INVALID_ARG;
    const int64_t G4 = d.G / 4;
    if (G4 == 0) return EP_OK;
    if (!owner_grad || !aligned_to(owner_grad, 16)) return EP_ERR_INVALID_ARG;
    PeerGrads pg;
    memset(&pg, 0, sizeof pg);
    for (int r = 0; r < d.R; ++r) {
        if (!replica_grads->recv_x[r] || !aligned_to(replica_grads->recv_x[r], 16)) return EP_ERR_INVALID_ARG;
        pg.rep[r] = (const float4 *)replica_grads->recv_x[r];
    }
    const int grid = num_sms() * 8;
    const cudaError_t err =
        launch_pdl(k_reduce_peers, dim3(grid), dim3(kRedPeerThreads), 0, (cudaStream_t)stream, pg, (float4 *)owner_grad,
                   (const int32_t *)h->ws.red_experts, (const int32_t *)h->ws.red_count,
                   (const int32_t *)h->ws.red_list, (const int32_t *)h->ws.red_n, d.R, d.S, h->world_rank * d.g, d.g,
                   G4);
    return err == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

ep_status_t ep_prefetch_replica_weights_peers(ep_handle_t *h, const ep_peer_table_t *weights,
                                              int64_t bytes_per_expert, void *prefetch_slots, void *stream) {
    if (!h) return EP_ERR_INVALID_ARG;
    if (!h->d.balanced) return EP_ERR_UNSUPPORTED;
    if (h->planned != 2) return h->planned == 1 ? EP_ERR_UNSUPPORTED : EP_ERR_NOT_PLANNED;
    const Dims &d = h->d;
    ep_status_t s = check_table(h, weights, true);
    if (s != EP_OK) return s;
    if (bytes_per_expert <= 0 || bytes_per_expert % 16 != 0 || !prefetch_slots || !aligned_to(prefetch_slots, 16))
        return EP_ERR_INVALID_ARG;
    // (slot, 16 KB chunk) items are counted in 32 bits
    if ((bytes_per_expert / 16384 + 1) * (int64_t)d.S > INT32_MAX / 2) return EP_ERR_INVALID_ARG;
    PeerRows pw;
    fill_rows(weights, d.R, &pw);
    const int64_t V = bytes_per_expert / 16;
    const int grid = num_sms() * 8;
    const cudaError_t err =
        launch_pdl(k_prefetch_peers, dim3(grid), dim3(kCopyPeerThreads), 0, (cudaStream_t)stream, pw,
                   (uint4 *)prefetch_slots, (const int32_t *)h->ws.replica_expert, h->world_rank, d.S, d.g, V);
    return err == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

// ---- CUDA IPC ---------------------------------------------------------------

typedef int (*mem_range_fn)(uintptr_t *base, size_t *size, uintptr_t ptr);

ep_status_t ep_ipc_export(const void *dev_ptr, uint8_t handle[64], int64_t *offset) {
    if (!dev_ptr || !handle || !offset) return EP_ERR_INVALID_ARG;
    // the allocation's base, from the driver (cuMemGetAddressRange)
    static mem_range_fn range = nullptr;
    if (!range) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return EP_ERR_CUDA;
        range = (mem_range_fn)fn;
    }
    uintptr_t base = 0;
    size_t size = 0;
    if (range(&base, &size, (uintptr_t)dev_ptr) != 0) return EP_ERR_INVALID_ARG;
    cudaIpcMemHandle_t hd;
    if (cudaIpcGetMemHandle(&hd, (void *)base) != cudaSuccess) {
        cudaGetLastError();
        return EP_ERR_CUDA;
    }
    static_assert(sizeof(cudaIpcMemHandle_t) == 64, "a CUDA IPC handle is 64 bytes");
    memcpy(handle, &hd, 64);
    *offset = (int64_t)((uintptr_t)dev_ptr - base);
    return EP_OK;
}

ep_status_t ep_ipc_import(const uint8_t handle[64], int64_t offset, void **dev_ptr, void **base) {
    if (!handle || !dev_ptr || !base || offset < 0) return EP_ERR_INVALID_ARG;
    cudaIpcMemHandle_t hd;
    memcpy(&hd, handle, 64);
    void *b = nullptr;
    if (cudaIpcOpenMemHandle(&b, hd, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
        cudaGetLastError();
        return EP_ERR_CUDA;
    }
    *base = b;
    *dev_ptr = (char *)b + offset;
    return EP_OK;
}

ep_status_t ep_ipc_close(void *base) {
    if (!base) return EP_ERR_INVALID_ARG;
    return cudaIpcCloseMemHandle(base) == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

} // extern "C"
