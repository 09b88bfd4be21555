// noalloc.cu -- ep_route_noalloc: the routing pass (counts, stable slots,
// HT destination rows) for callers that cannot allocate device memory.
//
// Its scratch (per-pair packed ranks, per-tile counts, tile flags and the
// layout tables) lives in one file-scope __device__ array of fixed size, so
// the call itself allocates nothing. It launches the same routing kernels as
// ep_plan, with a workspace whose scratch points into that array and whose
// outputs point at the caller's buffers.
#include <string.h>

#include <atomic>

#include "ep_internal.cuh"

namespace epb {
namespace {

// Scratch shared by every ep_route_noalloc call on a device; every GPU that
// loads the library holds it until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[EP_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch per device, looked up once per device
// with that device current (host code cannot use the symbol itself); threads
// that race to look it up store the same address.
std::atomic<void *> g_scratch_ptr[64];

size_t al256(size_t n) { return (n + 255) & ~(size_t)255; }

// every int32 argument must be 4-byte aligned; a misaligned one is refused
// before anything is launched
bool aligned4(const void *p) { return ((uintptr_t)p & 3u) == 0; }

// Bytes of scratch the routing kernels need for these sizes (plain HT layout,
// one logical rank).
size_t scratch_need(const Dims &d) {
    const size_t i4 = sizeof(int32_t);
    return al256(i4 * (size_t)(d.L > 0 ? d.L : 1))                                   // packed
           + al256(i4 * (size_t)d.E * (d.ntiles > 0 ? d.ntiles : 1))                 // blk
           + al256(i4 * (size_t)d.E * (d.nhist > 0 ? d.nhist : 1))                   // blk_cta
           + al256(i4 * (size_t)(d.nhist > 0 ? d.nhist : 1))                         // tile_flags
           + 3 * al256(i4 * (size_t)d.E)                                             // recv_counts, base0, len0
           + 3 * al256(i4 * 2);                                                      // rank_load, rank_off, red_count
}

} // namespace
} // namespace epb

using namespace epb;

extern "C" ep_status_t ep_route_noalloc(const int32_t *topk_idx, int32_t num_tokens, int32_t topk,
                                        int32_t num_experts, int32_t *dest_row, int32_t *expert_counts,
                                        int32_t *flags, void *stream) {
    ep_config_t cfg;
    memset(&cfg, 0, sizeof cfg);
    cfg.num_tokens = num_tokens;
    cfg.hidden = 8; // routing does not depend on the row width
    cfg.num_experts = num_experts;
    cfg.topk = topk;
    cfg.num_ranks = 1;
    cfg.mode = EP_MODE_HT;
    Dims d;
    ep_status_t s = derive_dims(&cfg, &d);
    if (s != EP_OK) return s;
    if (!expert_counts || !flags || !aligned4(expert_counts) || !aligned4(flags)) return EP_ERR_INVALID_ARG;
    if (d.L > 0 && (!topk_idx || !dest_row || !aligned4(topk_idx) || !aligned4(dest_row))) return EP_ERR_INVALID_ARG;
    if (scratch_need(d) > (size_t)EP_NOALLOC_SCRATCH_BYTES) return EP_ERR_TOO_LARGE;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return EP_ERR_CUDA;
    void *base = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (!base) { // set-up: once per device, with that device current
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return EP_ERR_CUDA;
        }
        g_scratch_ptr[dev].store(p, std::memory_order_release);
        base = p;
    }

    // Every scratch word a kernel reads is written earlier in the same call
    // (packed and the tile counts by the histogram kernel, the tables by the
    // assignment kernel), so nothing needs clearing between calls.
    Workspace ws;
    memset(&ws, 0, sizeof ws);
    char *p = (char *)base;
    auto take = [&p](size_t n) {
        char *q = p;
        p += al256(n);
        return (int32_t *)q;
    };
    ws.packed = take(sizeof(int32_t) * (size_t)(d.L > 0 ? d.L : 1));
    ws.blk = take(sizeof(int32_t) * (size_t)d.E * (d.ntiles > 0 ? d.ntiles : 1));
    ws.blk_cta = take(sizeof(int32_t) * (size_t)d.E * (d.nhist > 0 ? d.nhist : 1));
    ws.tile_flags = (uint32_t *)take(sizeof(int32_t) * (size_t)(d.nhist > 0 ? d.nhist : 1));
    ws.recv_counts = take(sizeof(int32_t) * (size_t)d.E);
    ws.base0 = take(sizeof(int32_t) * (size_t)d.E);
    ws.len0 = take(sizeof(int32_t) * (size_t)d.E);
    ws.rank_load = take(sizeof(int32_t) * 2);
    ws.rank_off = take(sizeof(int32_t) * 2);
    ws.red_count = take(sizeof(int32_t) * 2);
    ws.dest_row = dest_row;
    ws.cnt = expert_counts;
    ws.flags = (uint32_t *)flags;
    if (launch_plan(d, ws, topk_idx, (cudaStream_t)stream) != cudaSuccess) return EP_ERR_CUDA;
    return EP_OK;
}
