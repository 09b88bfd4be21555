// ep_internal.cuh -- handle layout and kernel launchers shared by the .cu
// files of libep_b200 (not part of the public ABI; see include/ep.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "ep.h"

namespace epb {

// Routing: each warp of the histogram kernel owns a "warp tile" of
// consecutive (token, k) pairs; tiles grow with the batch so that there are
// at most about kMaxTiles of them.
constexpr int kMaxTilePairs = 2048;
constexpr int kMaxTiles = 1024;
constexpr int kRouteThreads = 256;
constexpr int kAssignPer = 4;             // pairs per thread of the assignment kernel
constexpr int kRouteWarps = kRouteThreads / 32;
constexpr int kRouteWarpsLog2 = 3;
constexpr int kPlanThreads = 1024;
constexpr int kMaxExperts = 4096;
constexpr int kMaxTopk = 32;
constexpr int kRouterMaxExperts = 1024;   // ep_router_topk keeps a token's logits in one warp's registers
constexpr int kMaxRouteSmem = 200 * 1024; // dynamic shared memory cap of the routing kernels
constexpr int kSmallMaxPairs = 1024;      // single-CTA routing up to this many pairs ...
constexpr int kSmallMaxExperts = 512;     // ... and experts (plain layouts)
constexpr int kSmallMaxPlanPairs = 1024;  // single-CTA routing with a balanced plan up to this many pairs
                                          // (beyond it the three kernels measured faster: 8192 pairs, 43 vs 54 us)
constexpr int kClusterThreads = 1024;     // one-launch cluster routing: threads per CTA, at most
constexpr int kClusterWarps = kClusterThreads / 32;
constexpr int kClusterMaxPairs = 32768;  // ... up to this many (token, k) pairs

// Device workspace of a handle: the routing state one ep_plan builds and the
// later calls of the same forward/backward pass read.
struct Workspace {
    int32_t *dest_row;       // [T*K]: receive-buffer row of each pair, -1 if none
    int32_t *src_row;        // [rows]: pair index of each targeted row (NULL: not kept)
    int32_t *packed;         // [T*K]: expert | rank-in-tile << 16, 0xffff if not routed
    int32_t *blk;            // [ntiles][E]: each tile's base within its CTA's tiles
    int32_t *blk_cta;        // [nhist][E]: per-CTA counts, then bases over CTAs
    uint32_t *tile_flags;    // [nhist]: status bits seen by each histogram CTA
    int32_t *cnt;            // [E]
    int32_t *recv_counts;    // [R*(g+S)] (HT) or [E] (LL)
    int32_t *rank_load;      // [R]
    int32_t *rank_off;       // [R+1]
    int32_t *replica_expert; // [max(R*S,1)]
    int32_t *slot_list;      // [max(R*S,1)]: the filled replica slots (r*S+s), ascending
    int32_t *slot_count;     // [1]
    int32_t *direct_n;       // [R]: direct-read pieces per rank (direct_overflow)
    int32_t *direct_expert;  // [R*E]: piece i of rank r at r*E+i
    int32_t *direct_start;   // [R*E]: first stable index it covers
    int32_t *direct_len;     // [R*E]
    int32_t *base0;          // [E]: row of stable index 0 of each expert (piece 0)
    int32_t *len0;           // [E]: stable indices [0, len0) live in piece 0
    int32_t *xoff;           // [E+1]: extra pieces of expert e: [xoff[e], xoff[e+1])
    int32_t *xstart;         // [nx_max]: first stable index of an extra piece
    int32_t *xlen;           // [nx_max]
    int32_t *xdst;           // [nx_max]: row of the extra piece's first index
    int32_t *red_list;       // [E][R]: slots (r*S+s) holding e, ascending
    int32_t *red_n;          // [E]
    int32_t *red_experts;    // [E]: experts with at least one replica
    int32_t *red_count;      // [1]
    uint32_t *flags;         // [1]: EP_FLAG_* bits of the last plan
    unsigned long long *ticket; // [1]: CTAs of the scan kernel that have finished
    int32_t *jbase;          // [E]: world plan: this rank's first stable index within each expert
};

struct Dims {
    int T, H, E, K, R, g, S; // S = replica slots per rank (0 without a plan)
    int mode, cap, fp8, balanced, direct;
    int64_t L;               // T*K pairs
    int64_t rows;            // receive-buffer rows
    int64_t G;               // replica-gradient elements per expert
    int wt, wt_log2;         // pairs per warp tile (a power of two, >= 128)
    int ntiles, nhist;       // warp tiles, histogram CTAs
    int nassign;             // CTAs of the slot-assignment kernel
    int cl_size, cl_ppw;     // cluster routing: CTAs (8 or 16, 0 = not used), pairs per warp
    int cl_warps;            // cluster routing: warps per CTA (16 or 32)
    int nx_max;              // bound on extra pieces (R*S + E with a plan, else 0)
    int counts_len;          // recv_counts entries
    int world;               // 1: the routing completes a world plan (global rows, see ep_plan_world)
};

// Sizes derived from a validated configuration; also used by the host-only
// queries, so it allocates nothing.
ep_status_t derive_dims(const ep_config_t *cfg, Dims *d);
size_t workspace_bytes(const Dims &d);
void carve_workspace(const Dims &d, void *base, Workspace *ws);

// shared-memory needs of the routing kernels (host side, for validation)
size_t route_smem_layout(const Dims &d);
size_t route_smem_assign(const Dims &d);
size_t route_smem_hist(const Dims &d);
size_t route_smem_small(const Dims &d);
size_t route_smem_cluster(const Dims &d);
bool route_use_small(const Dims &d);
bool route_use_cluster(const Dims &d);
int plan_launches(const Dims &d);

// ---- launchers (each returns the launch's cudaError_t) ----
cudaError_t launch_plan(const Dims &d, const Workspace &ws, const int32_t *topk_idx, cudaStream_t st);
// world mode (ep_plan_local_counts / ep_plan_world)
cudaError_t launch_plan_local_counts(const Dims &d, const Workspace &ws, const int32_t *topk_idx, cudaStream_t st);
cudaError_t launch_plan_world(const Dims &d, const Workspace &ws, const int32_t *world_counts, int rank,
                              cudaStream_t st);
size_t route_smem_world(const Dims &d);
cudaError_t launch_dispatch(const Dims &d, const Workspace &ws, const void *x, const int32_t *topk_idx,
                            const float *topk_w, void *recv_x, float *recv_scales, float *recv_w,
                            int32_t *recv_expert, int32_t *recv_counts, cudaStream_t st);
cudaError_t launch_combine_backward(const Dims &d, const Workspace &ws, const void *grad_out, const float *topk_w,
                                    void *grad_expert_out, cudaStream_t st);
cudaError_t launch_combine(const Dims &d, const Workspace &ws, const void *y, const float *topk_w, void *out,
                           cudaStream_t st);
cudaError_t launch_prefetch(const Dims &d, const Workspace &ws, const void *weights, int64_t bytes_per_expert,
                            void *slots, cudaStream_t st);
cudaError_t launch_replica_reduce(const Dims &d, const Workspace &ws, const float *rep, float *owner,
                                  cudaStream_t st);

int num_sms();
// row movers' launch shape: vectors per thread and threads per CTA for a row
// part of n 16-byte vectors; vectors per row part for T rows of nvec vectors
void pick_shape(int n, int *per_thread, int *threads);
int row_part(int T, int nvec);

// Programmatic dependent launch: every kernel of the library waits for the
// grid before it in the stream to complete (and its writes to be visible)
// before touching memory, so its launch overlaps the previous kernel's tail.
// The short routing kernels also let the next grid launch as soon as all of
// their CTAs run; the long row movers do not (their grids span many waves,
// and an early launch of the next grid measured slower there).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

} // namespace epb

struct ep_handle {
    ep_config_t cfg;
    epb::Dims d;
    epb::Workspace ws;
    void *base;
    int device;
    int planned;       // 0 none, 1 ep_plan (single-GPU layout), 2 ep_plan_world (global rows)
    int counts_ready;  // ep_plan_local_counts ran since the last plan
    int world_rank;    // this handle's rank in its world plan
};
