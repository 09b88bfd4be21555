// data.cu -- the HBM-bound row movers: dispatch (bf16 copy or fused FP8
// cast), combine (gather + fp32 weighted reduce), their backward twins, and
// the replica-gradient reduce.
//
// NCCL EP paper (arXiv 2603.13606): dispatch takes tokens, top-k ids and
// weights and a handle, and yields received rows, ids and weights (Table V);
// FP8 quantization scales as a tensor role (Table IV); combine collects each
// token's expert results and sums them back into that token's row (Table II),
// per token at the receiver (Table III); the backward
// pass reuses the forward routing state (Fig. 5). MoonEP article, para. 5:
// gradients of duplicated experts pass through a reduce buffer and are added
// into the owner's gradients.
//
// Every kernel is a streaming row mover: one CTA per token row (or part of
// one), each input row read once and each output row written once, so the
// bytes moved are the algorithmic bytes. The bf16 dispatch moves its rows with
// bulk copies (the TMA engine) through shared memory; the others use 16-byte
// vector loads and stores from registers.
#include <cuda_bf16.h>

#include "bulk.cuh"
#include "ep_internal.cuh"
#include "rows.cuh"

namespace epb {
namespace {

__device__ __forceinline__ void stage_routing(const int32_t *__restrict__ dest_row, const float *__restrict__ w,
                                              int64_t pb, int K, int *s_dest, float *s_w) {
    if (threadIdx.x < K) {
        s_dest[threadIdx.x] = dest_row[pb + threadIdx.x];
        if (s_w) s_w[threadIdx.x] = w ? w[pb + threadIdx.x] : 1.0f;
    }
}

// Bulk copies and their bounded mbarrier wait: bulk.cuh.
constexpr int kBulkSlabVectors = 2048; // 32 KB of shared memory per bulk-copy CTA


// ---------------------------------------------------------------------------
// dispatch, bf16 payload, by bulk copies: one warp per (row, part); lane 0
// loads the part into shared memory (before griddepcontrol.wait, as in
// read_before_wait) and stores it to the K destination rows, a slab of at most
// `slab` bytes at a time. The other lanes stage the routing.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(32) k_dispatch_bulk(const uint8_t *__restrict__ x, const int32_t *__restrict__ idx,
                                                      const float *__restrict__ w,
                                                      const int32_t *__restrict__ dest_row, int K, int row_bytes,
                                                      int part_bytes, int slab, uint8_t *__restrict__ recv,
                                                      float *__restrict__ recv_w, int32_t *__restrict__ recv_expert,
                                                      const int32_t *__restrict__ counts_src,
                                                      int32_t *__restrict__ counts_dst, int counts_len,
                                                      uint32_t *__restrict__ status) {
    extern __shared__ __align__(128) uint8_t s_row[];
    __shared__ __align__(8) uint64_t s_bar;
    __shared__ int s_dest[kMaxTopk];
    const int t = blockIdx.x, lane = threadIdx.x;
    const int cb = blockIdx.y * part_bytes, n = min(part_bytes, row_bytes - cb); // this CTA's bytes of the row
    const uint8_t *src = x + (int64_t)t * row_bytes + cb;
    if (lane == 0) {
        mbar_init(&s_bar);
        bulk_load(s_row, src, (uint32_t)min(n, slab), &s_bar);
    }
    pdl_wait(); // no early trigger: measured slower for these multi-wave grids
    const int64_t pb = (int64_t)t * K;
    if (lane < K) {
        const int dr = dest_row[pb + lane];
        s_dest[lane] = dr;
        if (dr >= 0 && blockIdx.y == 0) {
            if (recv_w) recv_w[dr] = w[pb + lane];
            if (recv_expert) recv_expert[dr] = idx[pb + lane];
        }
    }
    if (t == 0 && blockIdx.y == 0 && counts_dst)
        for (int i = lane; i < counts_len; i += 32) counts_dst[i] = counts_src[i];
    __syncwarp();
    if (lane != 0) return;
    uint32_t parity = 0;
    for (int off = 0; off < n; off += slab, parity ^= 1u) {
        const int len = min(slab, n - off);
        if (off > 0) bulk_load(s_row, src + off, (uint32_t)len, &s_bar);
        if (!mbar_wait(&s_bar, parity)) {
            atomicOr(status, EP_FLAG_WAIT_TIMEOUT);
            // The load in flight still writes s_row: stay resident (bounded,
            // up to 8 more waits of 2 s) so that its bytes cannot land in the
            // shared memory of a CTA that takes this one's place. Past that
            // the flag stands for the whole launch.
            for (int r = 0; r < 8 && !mbar_wait(&s_bar, parity); ++r) {
            }
            return;
        }
        const uint64_t pol = policy_evict_first();
        for (int k = 0; k < K; ++k) {
            const int dr = s_dest[k];
            if (dr < 0) continue;
            bulk_store(recv + (int64_t)dr * row_bytes + cb + off, s_row, (uint32_t)len, pol);
        }
        bulk_stores_read(); // before s_row is reloaded, and before the CTA exits
    }
}

// ---------------------------------------------------------------------------
// dispatch, FP8 payload: per 128-element block b of x[t],
//   s_b = amax_b / 448, q = e4m3(x / s_b), all-zero block -> s = 0, q = +0.
// The cast is done once per token and its result stored K times.
// One thread owns 16 consecutive elements (two 16-byte loads, one 16-byte
// store); the 8 threads of a 128-block are 8 consecutive lanes.
// ---------------------------------------------------------------------------
// At least 5 CTAs per SM (48 registers) for up to two chunks a thread:
// measured faster than the unbounded 64-register build (HT prefill step
// 1016 -> 1011 us). Four and eight chunks a thread (rows of more than 8192
// elements) hold 2-4x the data in registers and would spill under that bound;
// they take 3 and 2 CTAs per SM.
constexpr int fp8_min_ctas(int cpt) { return cpt <= 2 ? 5 : cpt == 4 ? 3 : 2; }

template <int CPT>
__global__ void __launch_bounds__(256, fp8_min_ctas(CPT)) k_dispatch_fp8(const uint4 *__restrict__ x, const int32_t *__restrict__ idx,
                                                      const float *__restrict__ w,
                                                      const int32_t *__restrict__ dest_row, int K, int nchunk,
                                                      int part, uint4 *__restrict__ recv, float *__restrict__ scales,
                                                      float *__restrict__ recv_w, int32_t *__restrict__ recv_expert,
                                                      const int32_t *__restrict__ counts_src,
                                                      int32_t *__restrict__ counts_dst, int counts_len) {
    __shared__ int s_dest[kMaxTopk];
    const int t = blockIdx.x;
    const int64_t pb = (int64_t)t * K;
    const int nb = nchunk >> 3; // 128-element blocks per row
    // this CTA's chunks of the row (part is a multiple of 8: whole blocks)
    const int cb = blockIdx.y * part, n = min(part, nchunk - cb);
    const uint4 *src = x + (int64_t)t * 2 * nchunk + 2 * cb;
    const int step = CPT * blockDim.x;
    uint4 a[CPT], b[CPT];
    load_pairs<CPT>(src, 0, n, a, b); // before the wait: see read_before_wait
    pdl_wait(); // no early trigger: measured slower for these multi-wave grids
    if (threadIdx.x < K) {
        const int dr = dest_row[pb + threadIdx.x];
        s_dest[threadIdx.x] = dr;
        if (dr >= 0 && blockIdx.y == 0) {
            if (recv_w) recv_w[dr] = w[pb + threadIdx.x];
            if (recv_expert) recv_expert[dr] = idx[pb + threadIdx.x];
        }
    }
    if (t == 0 && blockIdx.y == 0 && counts_dst)
        for (int i = threadIdx.x; i < counts_len; i += blockDim.x) counts_dst[i] = counts_src[i];
    for (int c0 = 0; c0 < n; c0 += step) {
        if (c0 > 0) load_pairs<CPT>(src, c0, n, a, b);
        uint4 q[CPT];
        float sc[CPT];
#pragma unroll
        for (int i = 0; i < CPT; ++i) quant_chunk(a[i], b[i], q[i], sc[i]);
        if (c0 == 0) __syncthreads();
        for (int k = 0; k < K; ++k) {
            const int dr = s_dest[k];
            if (dr < 0) continue;
            uint4 *dst = recv + (int64_t)dr * nchunk + cb;
#pragma unroll
            for (int i = 0; i < CPT; ++i) {
                const int c = c0 + threadIdx.x + i * blockDim.x;
                if (c < n) {
                    dst[c] = q[i]; // write-back: measured faster here than st.global.cs
                    if ((c & 7) == 0) scales[(int64_t)dr * nb + ((cb + c) >> 3)] = sc[i];
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// combine: out[t] = bf16(fold_k fmaf(w[t,k], y[dest_row[t,k]], acc)), k in
// order, acc from +0; UNIT: unweighted fp32 sum (dispatch backward).
// ---------------------------------------------------------------------------
// At least 5 CTAs per SM (48 registers): measured faster than the unbounded
// 64-register build (HT prefill step 1025 -> 1014 us).
template <int CPT, bool UNIT, bool CS>
__global__ void __launch_bounds__(256, 5) k_combine(const uint4 *__restrict__ y, const float *__restrict__ w,
                                                 const int32_t *__restrict__ dest_row, int K, int nvec,
                                                 int part, uint4 *__restrict__ out) {
    pdl_wait(); // no early trigger: measured slower for these multi-wave grids
    __shared__ int s_dest[kMaxTopk];
    __shared__ float s_w[kMaxTopk];
    const int t = blockIdx.x;
    stage_routing(dest_row, w, (int64_t)t * K, K, s_dest, s_w);
    __syncthreads();
    const int cb = blockIdx.y * part, n = min(part, nvec - cb); // this CTA's vectors of the row
    const uint4 *yb = y + cb;
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
                    const int dr = k < K ? s_dest[k] : -1;
                    const uint4 *p = yb + (int64_t)dr * nvec + c;
                    v[kk] = dr >= 0 ? (CS ? __ldcs(p) : *p) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const int k = k0 + kk;
                    if (k >= K || s_dest[k] < 0) continue;
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
            out[(int64_t)t * nvec + cb + c] = pack8(acc); // write-back: measured faster than .cs
        }
    }
}

// ---------------------------------------------------------------------------
// combine backward: gy[dest_row[t,k]] = bf16(w[t,k] * g[t]) (fp32 product)
// ---------------------------------------------------------------------------
template <int VPT>
__global__ void __launch_bounds__(512) k_combine_bwd(const uint4 *__restrict__ g, const float *__restrict__ w,
                                                     const int32_t *__restrict__ dest_row, int K, int nvec,
                                                     int part, uint4 *__restrict__ gy) {
    pdl_wait(); // no early trigger: measured slower for these multi-wave grids
    __shared__ int s_dest[kMaxTopk];
    __shared__ float s_w[kMaxTopk];
    const int t = blockIdx.x;
    stage_routing(dest_row, w, (int64_t)t * K, K, s_dest, s_w);
    const int cb = blockIdx.y * part, n = min(part, nvec - cb); // this CTA's vectors of the row
    const uint4 *src = g + (int64_t)t * nvec + cb;
    const int step = VPT * blockDim.x;
    for (int c0 = 0; c0 < n; c0 += step) {
        uint4 v[VPT];
        load_slab<VPT>(src, c0, n, v);
        if (c0 == 0) __syncthreads();
        for (int k = 0; k < K; ++k) {
            const int dr = s_dest[k];
            if (dr < 0) continue;
            const float wk = s_w[k];
            uint4 *dst = gy + (int64_t)dr * nvec + cb;
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int c = c0 + threadIdx.x + i * blockDim.x;
                if (c >= n) continue;
                float f[8];
                unpack8(v[i], f);
#pragma unroll
                for (int u = 0; u < 8; ++u) f[u] = __fmul_rn(wk, f[u]);
                __stcs(dst + c, pack8(f));
            }
        }
    }
}

// ---------------------------------------------------------------------------
// replica-gradient reduce: owner[e] += rep[slot] for the slots holding e,
// ascending slot order, fp32. Persistent grid over (expert, chunk) items.
// ---------------------------------------------------------------------------
constexpr int kRedThreads = 256, kRedUnroll = 4;

__global__ void __launch_bounds__(kRedThreads) k_replica_reduce(const float4 *__restrict__ rep,
                                                                float4 *__restrict__ owner,
                                                                const int32_t *__restrict__ red_experts,
                                                                const int32_t *__restrict__ red_count,
                                                                const int32_t *__restrict__ red_list,
                                                                const int32_t *__restrict__ red_n, int R,
                                                                int64_t G4) {
    pdl_wait(); // no early trigger: measured slower for these multi-wave grids
    const int nred = *red_count;
    const int64_t chunk = (int64_t)kRedThreads * kRedUnroll;
    const int per = (int)((G4 + chunk - 1) / chunk); // chunks per expert (host-checked to fit)
    const int items = nred * per;
    for (int it = blockIdx.x; it < items; it += gridDim.x) {
        const int e = red_experts[it / per];
        const int64_t base = (int64_t)(it % per) * chunk + threadIdx.x;
        const int n = red_n[e];
        const int32_t *lst = red_list + (int64_t)e * R;
        float4 *o = owner + (int64_t)e * G4;
        float4 acc[kRedUnroll];
#pragma unroll
        for (int u = 0; u < kRedUnroll; ++u) {
            const int64_t i = base + (int64_t)u * kRedThreads;
            acc[u] = i < G4 ? o[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        for (int a = 0; a < n; ++a) {
            const float4 *r = rep + (int64_t)lst[a] * G4;
#pragma unroll
            for (int u = 0; u < kRedUnroll; ++u) {
                const int64_t i = base + (int64_t)u * kRedThreads;
                if (i < G4) {
                    const float4 v = __ldcs(r + i);
                    acc[u].x = __fadd_rn(acc[u].x, v.x);
                    acc[u].y = __fadd_rn(acc[u].y, v.y);
                    acc[u].z = __fadd_rn(acc[u].z, v.z);
                    acc[u].w = __fadd_rn(acc[u].w, v.w);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kRedUnroll; ++u) {
            const int64_t i = base + (int64_t)u * kRedThreads;
            if (i < G4) o[i] = acc[u];
        }
    }
}

// ---------------------------------------------------------------------------
// replica weight prefetch: slots[r*S+s] = weights[replica_expert[r*S+s]] for
// every filled slot. The grid strides over (slot, chunk) items of 8 KB, with
// twice the CTAs an SM holds: the CTAs that start late fill the SMs that
// finish early. Measured on the large step's plan (1.03 GB copied), 318 us
// against 331 us for 16 KB items on a grid that fits at once, and 325 us for
// 4 KB items.
// ---------------------------------------------------------------------------
constexpr int kCopyThreads = 256, kCopyUnroll = 2, kCopyCtasPerSm = 16;

__global__ void __launch_bounds__(kCopyThreads) k_prefetch(const uint4 *__restrict__ weights,
                                                           uint4 *__restrict__ slots,
                                                           const int32_t *__restrict__ replica_expert,
                                                           const int32_t *__restrict__ slot_list,
                                                           const int32_t *__restrict__ slot_count, int64_t V) {
    pdl_wait(); // no early trigger: measured slower for these multi-wave grids
    const int64_t chunk = (int64_t)kCopyThreads * kCopyUnroll;
    const int per = (int)((V + chunk - 1) / chunk); // chunks per expert (host-checked to fit)
    const int items = *slot_count * per;            // filled slots only
    for (int it = blockIdx.x; it < items; it += gridDim.x) {
        const int sl = slot_list[it / per];
        const int e = replica_expert[sl];
        const int64_t base = (int64_t)(it % per) * chunk + threadIdx.x;
        const uint4 *src = weights + (int64_t)e * V;
        uint4 *dst = slots + (int64_t)sl * V;
        uint4 v[kCopyUnroll];
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
            const int64_t i = base + (int64_t)u * kCopyThreads;
            if (i < V) v[u] = src[i];
        }
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
            const int64_t i = base + (int64_t)u * kCopyThreads;
            if (i < V) dst[i] = v[u];
        }
    }
}

#define EPB_SWITCH_VPT(v, KERNEL, ...)                                                                               \
    switch (v) {                                                                                                     \
    case 1: err = launch_pdl(KERNEL<1>, grid, dim3(threads), 0, st, __VA_ARGS__); break;                             \
    case 2: err = launch_pdl(KERNEL<2>, grid, dim3(threads), 0, st, __VA_ARGS__); break;                             \
    case 4: err = launch_pdl(KERNEL<4>, grid, dim3(threads), 0, st, __VA_ARGS__); break;                             \
    default: err = launch_pdl(KERNEL<8>, grid, dim3(threads), 0, st, __VA_ARGS__); break;                            \
    }

} // namespace

// vectors per thread and threads per CTA for a row of `n` 16-byte vectors
void pick_shape(int n, int *per_thread, int *threads) {
    for (int v = 1; v <= 8; v <<= 1) {
        const int th = ((n + v - 1) / v + 31) / 32 * 32;
        if (th <= 256) {
            *per_thread = v;
            *threads = th < 32 ? 32 : th;
            return;
        }
    }
    *per_thread = 8;
    *threads = 256; // rows longer than 2048 vectors loop over slabs
}

// Vectors of a row per CTA. A batch of a few thousand tokens gives a grid of
// one or two waves of one-row CTAs, whose last, partial wave leaves most SMs
// idle while it drains; such rows are cut into parts (whole warps of vectors,
// at least kSplitMinVectors each) until the grid has about kSplitCtasPerSm
// CTAs per SM. Large batches keep one CTA per row.
constexpr int kSplitCtasPerSm = 32, kSplitMinVectors = 64;

int row_part(int T, int nvec) {
    const int64_t want = (int64_t)kSplitCtasPerSm * num_sms();
    int parts = 1;
    while ((int64_t)T * parts < want && nvec / (2 * parts) >= kSplitMinVectors) parts *= 2;
    if (parts == 1) return nvec;
    return ((nvec + parts - 1) / parts + 31) / 32 * 32;
}

cudaError_t launch_dispatch(const Dims &d, const Workspace &ws, const void *x, const int32_t *topk_idx,
                            const float *topk_w, void *recv_x, float *recv_scales, float *recv_w,
                            int32_t *recv_expert, int32_t *recv_counts, cudaStream_t st) {
    if (d.T == 0) {
        if (recv_counts)
            return cudaMemcpyAsync(recv_counts, ws.recv_counts, sizeof(int32_t) * d.counts_len,
                                   cudaMemcpyDeviceToDevice, st);
        return cudaSuccess;
    }
    int per, threads;
    cudaError_t err = cudaSuccess;
    if (d.fp8) {
        const int nchunk = d.H / 16; // a multiple of 8, and so is every part
        const int part = row_part(d.T, nchunk);
        const dim3 grid(d.T, (nchunk + part - 1) / part);
        pick_shape(part, &per, &threads);
        EPB_SWITCH_VPT(per, k_dispatch_fp8, (const uint4 *)x, topk_idx, topk_w, ws.dest_row, d.K, nchunk, part,
                       (uint4 *)recv_x, recv_scales, recv_w, recv_expert, ws.recv_counts, recv_counts,
                       d.counts_len);
    } else {
        const int nvec = d.H / 8;
        const int part = row_part(d.T, nvec);
        const dim3 grid(d.T, (nvec + part - 1) / part);
        const int slab = min(part, kBulkSlabVectors) * 16;
        err = launch_pdl(k_dispatch_bulk, grid, dim3(32), (size_t)slab, st, (const uint8_t *)x, topk_idx, topk_w,
                         ws.dest_row, d.K, nvec * 16, part * 16, slab, (uint8_t *)recv_x, recv_w, recv_expert,
                         ws.recv_counts, recv_counts, d.counts_len, ws.flags);
    }
    return err;
}

cudaError_t launch_combine_backward(const Dims &d, const Workspace &ws, const void *grad_out, const float *topk_w,
                                    void *grad_expert_out, cudaStream_t st) {
    if (d.T == 0) return cudaSuccess;
    const int nvec = d.H / 8;
    const int part = row_part(d.T, nvec);
    const dim3 grid(d.T, (nvec + part - 1) / part);
    int per, threads;
    cudaError_t err = cudaSuccess;
    pick_shape(part, &per, &threads);
    // whole rows of 257..1024 vectors: two vectors a thread, up to 512 threads
    // (large training step 10.17 -> 10.10 ms against four vectors a thread)
    if (part == nvec && nvec > 256 && nvec <= 1024) {
        per = 2;
        threads = ((nvec + 1) / 2 + 31) / 32 * 32;
    }
    EPB_SWITCH_VPT(per, k_combine_bwd, (const uint4 *)grad_out, topk_w, ws.dest_row, d.K, nvec, part,
                   (uint4 *)grad_expert_out);
    return err;
}

cudaError_t launch_combine(const Dims &d, const Workspace &ws, const void *y, const float *topk_w, void *out,
                           cudaStream_t st) {
    if (d.T == 0) return cudaSuccess;
    const int nvec = d.H / 8;
    const int part = row_part(d.T, nvec);
    const dim3 grid(d.T, (nvec + part - 1) / part);
    int per, threads;
    pick_shape(part, &per, &threads);
    const uint4 *yy = (const uint4 *)y;
    uint4 *oo = (uint4 *)out;
    const dim3 block(threads);
    // Streaming (evict-first) loads measured faster when rows are cut into parts
    // (LL decode: combine 28.9 vs 31.7 us) and slower for whole rows (HT
    // prefill: 646 vs 619 us), so they are used only for parts.
    const bool cs = part < nvec;
    const float *none = nullptr;
#define EPB_COMBINE(C, U, S, W)                                                                                      \
    return launch_pdl(k_combine<C, U, S>, grid, block, 0, st, yy, W, ws.dest_row, d.K, nvec, part, oo)
#define EPB_COMBINE_CPT(U, S, W)                                                                                     \
    switch (per) {                                                                                                   \
    case 1: EPB_COMBINE(1, U, S, W);                                                                                 \
    case 2: EPB_COMBINE(2, U, S, W);                                                                                 \
    case 4: EPB_COMBINE(4, U, S, W);                                                                                 \
    default: EPB_COMBINE(8, U, S, W);                                                                                \
    }
    if (topk_w) {
        if (cs) EPB_COMBINE_CPT(false, true, topk_w)
        EPB_COMBINE_CPT(false, false, topk_w)
    }
    if (cs) EPB_COMBINE_CPT(true, true, none)
    EPB_COMBINE_CPT(true, false, none)
#undef EPB_COMBINE_CPT
#undef EPB_COMBINE
}

cudaError_t launch_prefetch(const Dims &d, const Workspace &ws, const void *weights, int64_t bytes_per_expert,
                            void *slots, cudaStream_t st) {
    const int64_t V = bytes_per_expert / 16;
    if (V == 0 || d.R * d.S == 0) return cudaSuccess;
    const int grid = num_sms() * kCopyCtasPerSm;
    return launch_pdl(k_prefetch, dim3(grid), dim3(kCopyThreads), 0, st, (const uint4 *)weights, (uint4 *)slots,
                      (const int32_t *)ws.replica_expert, (const int32_t *)ws.slot_list,
                      (const int32_t *)ws.slot_count, V);
}

cudaError_t launch_replica_reduce(const Dims &d, const Workspace &ws, const float *rep, float *owner,
                                  cudaStream_t st) {
    const int64_t G4 = d.G / 4;
    if (G4 == 0) return cudaSuccess;
    const int grid = num_sms() * 8;
    return launch_pdl(k_replica_reduce, dim3(grid), dim3(kRedThreads), 0, st, (const float4 *)rep, (float4 *)owner,
                      (const int32_t *)ws.red_experts, (const int32_t *)ws.red_count, (const int32_t *)ws.red_list,
                      (const int32_t *)ws.red_n, d.R, G4);
}

} // namespace epb
