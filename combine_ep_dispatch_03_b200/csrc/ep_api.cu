// ep_api.cu -- the C ABI declared in include/ep.h: argument checks, the
// handle's one-time workspace, and the stream-ordered launches.
#include <stdlib.h>
#include <string.h>

#include <atomic>

#include "ep_internal.cuh"

namespace epb {

int num_sms() {
    // per device, filled on first use; threads that race to fill it store the same value
    static std::atomic<int> cached[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

ep_status_t derive_dims(const ep_config_t *c, Dims *d) {
    if (!c || !d) return EP_ERR_INVALID_ARG;
    const int T = c->num_tokens, H = c->hidden, E = c->num_experts, K = c->topk, R = c->num_ranks;
    if (T < 0 || H <= 0 || H % 8 != 0 || E < 1 || E > kMaxExperts || K < 1 || K > kMaxTopk || K > E || R < 1 ||
        E % R != 0)
        return EP_ERR_INVALID_ARG;
    if (c->mode != EP_MODE_LL && c->mode != EP_MODE_HT) return EP_ERR_INVALID_ARG;
    if (c->fp8 != 0 && c->fp8 != 1) return EP_ERR_INVALID_ARG;
    if (c->balanced != 0 && c->balanced != 1) return EP_ERR_INVALID_ARG;
    if (c->direct_overflow != 0 && (c->direct_overflow != 1 || !c->balanced)) return EP_ERR_INVALID_ARG;
    if (c->fp8 && H % 128 != 0) return EP_ERR_INVALID_ARG;
    if (c->grad_elems_per_expert < 0 || c->grad_elems_per_expert % 4 != 0) return EP_ERR_INVALID_ARG;
    // the reduce walks (expert, 4096-element chunk) items with 32-bit counters
    if ((c->grad_elems_per_expert / 4096 + 1) * (int64_t)c->num_experts > INT32_MAX / 2) return EP_ERR_INVALID_ARG;
    const int g = E / R;
    const int64_t L = (int64_t)T * K;
    if (L > INT32_MAX / 2) return EP_ERR_INVALID_ARG;
    memset(d, 0, sizeof *d);
    d->T = T; d->H = H; d->E = E; d->K = K; d->R = R; d->g = g;
    d->mode = c->mode; d->fp8 = c->fp8; d->balanced = c->balanced; d->direct = c->direct_overflow;
    d->L = L;
    d->G = c->grad_elems_per_expert;
    if (c->mode == EP_MODE_LL) {
        if (c->balanced) return EP_ERR_UNSUPPORTED; // the plan is an HT (training / prefill) feature
        if (c->ll_capacity < 1) return EP_ERR_INVALID_ARG;
        if ((int64_t)E * c->ll_capacity > INT32_MAX / 2) return EP_ERR_INVALID_ARG;
        d->cap = c->ll_capacity;
        d->rows = (int64_t)E * c->ll_capacity;
        d->counts_len = E;
    } else {
        d->rows = L;
        if (c->balanced) {
            const int S = c->replica_slots == 0 ? g : c->replica_slots;
            if (S < 1 || S > g) return EP_ERR_INVALID_ARG;
            d->S = S;
        } else if (c->replica_slots != 0) {
            return EP_ERR_INVALID_ARG;
        }
        d->counts_len = R * (g + d->S);
    }
    // pieces beyond each expert's own rows: replica slots, tails, and direct
    // pieces (each of which ends an expert or exhausts a receiver)
    d->nx_max = c->balanced ? R * d->S + 2 * E + R : 0;
    d->wt_log2 = 7; // tiles of 2^7 .. 2^11 pairs, at most about kMaxTiles of them
    while ((1 << d->wt_log2) < kMaxTilePairs && ((int64_t)kMaxTiles << d->wt_log2) < L) ++d->wt_log2;
    d->wt = 1 << d->wt_log2;
    d->ntiles = (int)((L + d->wt - 1) / d->wt);
    d->nhist = (d->ntiles + kRouteWarps - 1) / kRouteWarps;
    const int64_t per_cta = (int64_t)kRouteThreads * kAssignPer; // pairs per assignment CTA
    d->nassign = (int)(L > 0 ? (L + per_cta - 1) / per_cta : 1);
    // cluster routing: at most kClusterMaxPairs pairs (measured faster than
    // the three-kernel path there, slower beyond); with a balanced plan, every
    // CTA of the cluster runs the planner after the cluster barrier. The
    // cluster shape keeps each warp near 64 pairs with as few warps per SM as
    // that allows, since the warp votes of the first pass issue slowly when
    // every warp of an SM votes. Step times measured per shape: 8192 pairs,
    // 8 CTAs x 16 warps 48.5 us (x 32 warps 49.0); 16384 pairs, 16 x 16
    // 53.5 us (8 x 32 54.9); 32768 pairs, 16 x 32 105.6 us (16 x 16 106.5).
    if (L <= kClusterMaxPairs) {
        const int cs = L > 8192 ? 16 : 8, cw = L > 16384 ? 32 : 16;
        const int64_t ppw = ((L + (int64_t)cs * cw - 1) / ((int64_t)cs * cw) + 31) / 32 * 32;
        d->cl_size = cs;
        d->cl_warps = cw;
        d->cl_ppw = (int)(ppw > 0 ? ppw : 32);
        if (route_smem_cluster(*d) > (size_t)kMaxRouteSmem) d->cl_size = 0;
    }
    // the routing kernels keep their tables in one CTA's shared memory
    if (route_smem_layout(*d) > (size_t)kMaxRouteSmem || route_smem_assign(*d) > (size_t)kMaxRouteSmem ||
        route_smem_hist(*d) > (size_t)kMaxRouteSmem)
        return EP_ERR_UNSUPPORTED;
    return EP_OK;
}

static size_t align256(size_t n) { return (n + 255) & ~(size_t)255; }

// every array is placed on a 256-byte boundary
#define EPB_WS_FIELDS(X)                                                                                             \
    X(dest_row, d.L > 0 ? d.L : 1)                                                                                    \
    X(src_row, d.rows > 0 ? d.rows : 1)                                                                               \
    X(packed, d.L > 0 ? d.L : 1)                                                                                      \
    X(blk, (int64_t)d.E * (d.ntiles > 0 ? d.ntiles : 1))                                                              \
    X(blk_cta, (int64_t)d.E * (d.nhist > 0 ? d.nhist : 1))                                                            \
    X(tile_flags, d.nhist > 0 ? d.nhist : 1)                                                                          \
    X(cnt, d.E)                                                                                                       \
    X(recv_counts, d.counts_len)                                                                                      \
    X(rank_load, d.R)                                                                                                 \
    X(rank_off, d.R + 1)                                                                                              \
    X(replica_expert, d.R *(d.S > 0 ? d.S : 1))                                                                       \
    X(slot_list, d.R *(d.S > 0 ? d.S : 1))                                                                            \
    X(slot_count, 1)                                                                                                  \
    X(direct_n, d.R)                                                                                                  \
    X(direct_expert, d.direct ? (int64_t)d.R * d.E : 1)                                                               \
    X(direct_start, d.direct ? (int64_t)d.R * d.E : 1)                                                                \
    X(direct_len, d.direct ? (int64_t)d.R * d.E : 1)                                                                  \
    X(base0, d.E)                                                                                                     \
    X(len0, d.E)                                                                                                      \
    X(xoff, d.E + 1)                                                                                                  \
    X(xstart, d.nx_max > 0 ? d.nx_max : 1)                                                                            \
    X(xlen, d.nx_max > 0 ? d.nx_max : 1)                                                                              \
    X(xdst, d.nx_max > 0 ? d.nx_max : 1)                                                                              \
    X(red_list, (int64_t)d.E * d.R)                                                                                   \
    X(red_n, d.E)                                                                                                     \
    X(red_experts, d.E)                                                                                               \
    X(red_count, 1)                                                                                                   \
    X(flags, 1)                                                                                                       \
    X(ticket, 2)                                                                                                      \
    X(jbase, d.E)

size_t workspace_bytes(const Dims &d) {
    size_t n = 0;
#define EPB_SIZE(name, count) n += align256(sizeof(int32_t) * (size_t)(count));
    EPB_WS_FIELDS(EPB_SIZE)
#undef EPB_SIZE
    return n;
}

void carve_workspace(const Dims &d, void *base, Workspace *ws) {
    char *p = (char *)base;
#define EPB_CARVE(name, count)                                                                                       \
    ws->name = (decltype(ws->name))p;                                                                                 \
    p += align256(sizeof(int32_t) * (size_t)(count));
    EPB_WS_FIELDS(EPB_CARVE)
#undef EPB_CARVE
}

} // namespace epb

using namespace epb;

static inline cudaStream_t as_stream(void *s) { return (cudaStream_t)s; }
static inline bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

extern "C" {

ep_status_t ep_validate_config(const ep_config_t *cfg) {
    Dims d;
    return derive_dims(cfg, &d);
}

ep_status_t ep_recv_rows(const ep_config_t *cfg, int64_t *rows) {
    Dims d;
    if (!rows) return EP_ERR_INVALID_ARG;
    const ep_status_t s = derive_dims(cfg, &d);
    if (s != EP_OK) return s;
    *rows = d.rows;
    return EP_OK;
}

ep_status_t ep_output_shape(const ep_config_t *cfg, int64_t dims[4], int32_t *ndim) {
    Dims d;
    if (!dims || !ndim) return EP_ERR_INVALID_ARG;
    const ep_status_t s = derive_dims(cfg, &d);
    if (s != EP_OK) return s;
    if (d.mode == EP_MODE_LL) {
        *ndim = 4;
        dims[0] = d.R;
        dims[1] = d.g;
        dims[2] = d.cap;
        dims[3] = d.H;
    } else {
        *ndim = 2;
        dims[0] = d.rows;
        dims[1] = d.H;
        dims[2] = 1;
        dims[3] = 1;
    }
    return EP_OK;
}

ep_status_t ep_recv_counts_len(const ep_config_t *cfg, int64_t *len) {
    Dims d;
    if (!len) return EP_ERR_INVALID_ARG;
    const ep_status_t s = derive_dims(cfg, &d);
    if (s != EP_OK) return s;
    *len = d.counts_len;
    return EP_OK;
}

ep_status_t ep_workspace_bytes(const ep_config_t *cfg, size_t *bytes) {
    Dims d;
    if (!bytes) return EP_ERR_INVALID_ARG;
    const ep_status_t s = derive_dims(cfg, &d);
    if (s != EP_OK) return s;
    *bytes = workspace_bytes(d);
    return EP_OK;
}

ep_status_t ep_plan_kernel_count(const ep_config_t *cfg, int32_t *count) {
    Dims d;
    if (!count) return EP_ERR_INVALID_ARG;
    const ep_status_t s = derive_dims(cfg, &d);
    if (s != EP_OK) return s;
    *count = plan_launches(d);
    return EP_OK;
}

const char *ep_version(void) { return "0.1.0"; }

const char *ep_status_string(ep_status_t s) {
    switch (s) {
    case EP_OK: return "EP_OK";
    case EP_ERR_INVALID_ARG: return "EP_ERR_INVALID_ARG";
    case EP_ERR_CUDA: return "EP_ERR_CUDA";
    case EP_ERR_UNSUPPORTED: return "EP_ERR_UNSUPPORTED";
    case EP_ERR_NOT_PLANNED: return "EP_ERR_NOT_PLANNED";
    case EP_ERR_NO_MEMORY: return "EP_ERR_NO_MEMORY";
    case EP_ERR_TOO_LARGE: return "EP_ERR_TOO_LARGE";
    }
    return "EP_ERR_UNKNOWN";
}

ep_status_t ep_create(const ep_config_t *cfg, ep_handle_t **out) {
    if (!out) return EP_ERR_INVALID_ARG;
    *out = nullptr;
    Dims d;
    ep_status_t s = derive_dims(cfg, &d);
    if (s != EP_OK) return s;
    ep_handle_t *h = (ep_handle_t *)calloc(1, sizeof(ep_handle_t));
    if (!h) return EP_ERR_NO_MEMORY;
    h->cfg = *cfg;
    h->d = d;
    if (cudaGetDevice(&h->device) != cudaSuccess) {
        free(h);
        return EP_ERR_CUDA;
    }
    const size_t bytes = workspace_bytes(d);
    if (cudaMalloc(&h->base, bytes) != cudaSuccess) {
        cudaGetLastError();
        free(h);
        return EP_ERR_NO_MEMORY;
    }
    carve_workspace(d, h->base, &h->ws);
    if (cudaMemset(h->base, 0, bytes) != cudaSuccess) {
        cudaFree(h->base);
        free(h);
        return EP_ERR_CUDA;
    }
    *out = h;
    return EP_OK;
}

ep_status_t ep_destroy(ep_handle_t *h) {
    if (!h) return EP_OK;
    int prev = 0;
    cudaGetDevice(&prev);
    cudaSetDevice(h->device);
    cudaDeviceSynchronize();
    const cudaError_t e = cudaFree(h->base);
    cudaSetDevice(prev);
    free(h);
    return e == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

ep_status_t ep_plan(ep_handle_t *h, const int32_t *topk_idx, void *stream) {
    if (!h) return EP_ERR_INVALID_ARG;
    if (h->d.T > 0 && (!topk_idx || !aligned(topk_idx, 4))) return EP_ERR_INVALID_ARG;
    h->counts_ready = 0;
    if (launch_plan(h->d, h->ws, topk_idx, as_stream(stream)) != cudaSuccess) return EP_ERR_CUDA;
    h->planned = 1;
    return EP_OK;
}

ep_status_t ep_dispatch(ep_handle_t *h, const void *x, const int32_t *topk_idx, const float *topk_w, void *recv_x,
                        float *recv_scales, float *recv_w, int32_t *recv_expert, int32_t *recv_counts,
                        void *stream) {
    if (!h) return EP_ERR_INVALID_ARG;
    if (!h->planned) return EP_ERR_NOT_PLANNED;
    if (h->planned == 2) return EP_ERR_UNSUPPORTED; // rows are global: the peer calls
    const Dims &d = h->d;
    if (d.T > 0) {
        if (!x || !recv_x || !aligned(x, 16) || !aligned(recv_x, 16)) return EP_ERR_INVALID_ARG;
        if (recv_w && (!topk_w || !aligned(topk_w, 4) || !aligned(recv_w, 4))) return EP_ERR_INVALID_ARG;
        if (recv_expert && (!topk_idx || !aligned(topk_idx, 4) || !aligned(recv_expert, 4)))
            return EP_ERR_INVALID_ARG;
        if (d.fp8 && (!recv_scales || !aligned(recv_scales, 4))) return EP_ERR_INVALID_ARG;
    }
    if (!d.fp8 && recv_scales) return EP_ERR_INVALID_ARG;
    if (recv_counts && !aligned(recv_counts, 4)) return EP_ERR_INVALID_ARG;
    if (launch_dispatch(d, h->ws, x, topk_idx, topk_w, recv_x, recv_scales, recv_w, recv_expert, recv_counts,
                        as_stream(stream)) != cudaSuccess)
        return EP_ERR_CUDA;
    return EP_OK;
}

ep_status_t ep_combine(ep_handle_t *h, const void *expert_out, const float *topk_w, void *out, void *stream) {
    if (!h) return EP_ERR_INVALID_ARG;
    if (!h->planned) return EP_ERR_NOT_PLANNED;
    if (h->planned == 2) return EP_ERR_UNSUPPORTED; // rows are global: the peer calls
    if (h->d.T > 0 && (!expert_out || !topk_w || !out || !aligned(expert_out, 16) || !aligned(out, 16) ||
                       !aligned(topk_w, 4)))
        return EP_ERR_INVALID_ARG;
    if (launch_combine(h->d, h->ws, expert_out, topk_w, out, as_stream(stream)) != cudaSuccess) return EP_ERR_CUDA;
    return EP_OK;
}

ep_status_t ep_combine_backward(ep_handle_t *h, const void *grad_out, const float *topk_w, void *grad_expert_out,
                                void *stream) {
    if (!h) return EP_ERR_INVALID_ARG;
    if (!h->planned) return EP_ERR_NOT_PLANNED;
    if (h->planned == 2) return EP_ERR_UNSUPPORTED; // rows are global: the peer calls
    if (h->d.T > 0 && (!grad_out || !topk_w || !grad_expert_out || !aligned(grad_out, 16) ||
                       !aligned(grad_expert_out, 16) || !aligned(topk_w, 4)))
        return EP_ERR_INVALID_ARG;
    if (launch_combine_backward(h->d, h->ws, grad_out, topk_w, grad_expert_out, as_stream(stream)) != cudaSuccess)
        return EP_ERR_CUDA;
    return EP_OK;
}

ep_status_t ep_dispatch_backward(ep_handle_t *h, const void *grad_recv, void *grad_x, void *stream) {
    if (!h) return EP_ERR_INVALID_ARG;
    if (!h->planned) return EP_ERR_NOT_PLANNED;
    if (h->planned == 2) return EP_ERR_UNSUPPORTED; // rows are global: the peer calls
    if (h->d.T > 0 && (!grad_recv || !grad_x || !aligned(grad_recv, 16) || !aligned(grad_x, 16)))
        return EP_ERR_INVALID_ARG;
    if (launch_combine(h->d, h->ws, grad_recv, nullptr, grad_x, as_stream(stream)) != cudaSuccess)
        return EP_ERR_CUDA;
    return EP_OK;
}

ep_status_t ep_reduce_replica_grads(ep_handle_t *h, const float *replica_grad, float *owner_grad, void *stream) {
    if (!h) return EP_ERR_INVALID_ARG;
    if (!h->d.balanced) return EP_ERR_UNSUPPORTED;
    if (!h->planned) return EP_ERR_NOT_PLANNED;
    if (h->planned == 2) return EP_ERR_UNSUPPORTED; // rows are global: the peer calls
    if (h->d.G > 0 && (!replica_grad || !owner_grad || !aligned(replica_grad, 16) || !aligned(owner_grad, 16)))
        return EP_ERR_INVALID_ARG;
    if (launch_replica_reduce(h->d, h->ws, replica_grad, owner_grad, as_stream(stream)) != cudaSuccess)
        return EP_ERR_CUDA;
    return EP_OK;
}

ep_status_t ep_prefetch_replica_weights(ep_handle_t *h, const void *expert_weights, int64_t bytes_per_expert,
                                        void *prefetch_slots, void *stream) {
    if (!h) return EP_ERR_INVALID_ARG;
    if (!h->d.balanced) return EP_ERR_UNSUPPORTED;
    if (!h->planned) return EP_ERR_NOT_PLANNED;
    if (h->planned == 2) return EP_ERR_UNSUPPORTED; // rows are global: the peer calls
    if (bytes_per_expert <= 0 || bytes_per_expert % 16 != 0 || !expert_weights || !prefetch_slots ||
        !aligned(expert_weights, 16) || !aligned(prefetch_slots, 16))
        return EP_ERR_INVALID_ARG;
    // (slot, 8 KB chunk) items are counted in 32 bits
    if ((bytes_per_expert / 8192 + 1) * (int64_t)h->d.R * h->d.S > INT32_MAX / 2) return EP_ERR_INVALID_ARG;
    if (launch_prefetch(h->d, h->ws, expert_weights, bytes_per_expert, prefetch_slots, as_stream(stream)) !=
        cudaSuccess)
        return EP_ERR_CUDA;
    return EP_OK;
}

ep_status_t ep_get_plan(ep_handle_t *h, int32_t *replica_expert_host, int32_t *rank_load_host, void *stream) {
    if (!h) return EP_ERR_INVALID_ARG;
    if (!h->planned) return EP_ERR_NOT_PLANNED;
    if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return EP_ERR_CUDA;
    // without a plan there are no slots (R*S = 0) and nothing is written
    if (replica_expert_host && h->d.S > 0 &&
        cudaMemcpy(replica_expert_host, h->ws.replica_expert, sizeof(int32_t) * h->d.R * h->d.S,
                   cudaMemcpyDeviceToHost) != cudaSuccess)
        return EP_ERR_CUDA;
    if (rank_load_host &&
        cudaMemcpy(rank_load_host, h->ws.rank_load, sizeof(int32_t) * h->d.R, cudaMemcpyDeviceToHost) != cudaSuccess)
        return EP_ERR_CUDA;
    return EP_OK;
}

ep_status_t ep_get_status(ep_handle_t *h, int32_t *flags, void *stream) {
    if (!h || !flags) return EP_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return EP_ERR_CUDA;
    uint32_t f = 0;
    if (cudaMemcpy(&f, h->ws.flags, sizeof f, cudaMemcpyDeviceToHost) != cudaSuccess) return EP_ERR_CUDA;
    *flags = (int32_t)f;
    return EP_OK;
}

ep_status_t ep_get_tensor(const ep_handle_t *h, ep_tensor_t which, const void **dptr, int64_t *numel) {
    if (!h || !dptr || !numel) return EP_ERR_INVALID_ARG;
    const Dims &d = h->d;
    switch (which) {
    case EP_T_DEST_ROW: *dptr = h->ws.dest_row; *numel = d.L; break;
    case EP_T_EXPERT_COUNTS: *dptr = h->ws.cnt; *numel = d.E; break;
    case EP_T_RECV_COUNTS: *dptr = h->ws.recv_counts; *numel = d.counts_len; break;
    case EP_T_RANK_LOAD: *dptr = h->ws.rank_load; *numel = d.R; break;
    case EP_T_RANK_OFFSET: *dptr = h->ws.rank_off; *numel = d.R + 1; break;
    case EP_T_REPLICA_EXPERT: *dptr = h->ws.replica_expert; *numel = (int64_t)d.R * d.S; break;
    case EP_T_DIRECT_COUNT: *dptr = h->ws.direct_n; *numel = d.direct ? d.R : 0; break;
    case EP_T_DIRECT_EXPERT: *dptr = h->ws.direct_expert; *numel = d.direct ? (int64_t)d.R * d.E : 0; break;
    case EP_T_DIRECT_LEN: *dptr = h->ws.direct_len; *numel = d.direct ? (int64_t)d.R * d.E : 0; break;
    case EP_T_SRC_ROW: *dptr = h->ws.src_row; *numel = d.rows; break;
    default: return EP_ERR_INVALID_ARG;
    }
    return EP_OK;
}

} // extern "C"
