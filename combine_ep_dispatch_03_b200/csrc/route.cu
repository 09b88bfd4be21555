// route.cu -- routing for one forward pass: per-expert counts, stable slots,
// the HT / LL layouts and the balanced-replica plan.
//
// NCCL EP paper (arXiv 2603.13606), Table III: HT output is "2D with token
// counts", LL output is "3D expert-major". MoonEP article, paras. 3-5: rows go
// straight to expert-grouped rank positions; a GPU planner replicates hot
// experts into at most E/R prefetch slots per rank so that every rank gets a
// predictable row count.
//
// Results are deterministic: positions come from counts and scans, never from
// the order in which atomics land.
//
// Large batches, three kernels:
//   k_route_hist    per warp tile of consecutive pairs: validate ids, give
//                   each pair its rank among the tile's pairs of the same
//                   expert (a ballot per id bit), count the tile's pairs
//                   per expert
//   k_route_scan    per expert: exclusive scan of the tile counts over tiles;
//                   with a balanced plan, the CTA that finishes last (a
//                   ticket counter, no waiting) builds the plan
//   k_route_assign  per pair: stable index j = tile base + rank in tile ->
//                   destination row through the layout tables (each CTA
//                   computes the plain layouts' expert offsets itself)
// Batches up to 32768 pairs, one kernel:
//   k_route_cluster a thread-block cluster of 8 or 16 CTAs; each CTA counts
//                   and ranks its share of the pairs in shared memory, stores
//                   its per-expert totals into every CTA's shared memory
//                   (distributed shared memory) before one cluster barrier,
//                   builds the layout (or the whole balanced plan) from the
//                   totals itself, and then assigns its own pairs; CTA 0
//                   also writes the tables out
// Tiny batches (with a plan, up to 1024 pairs), one kernel:
//   k_route_small   one CTA does all of the above in shared memory
#include <atomic>

#include <cooperative_groups.h>

#include "ep_internal.cuh"

namespace cg = cooperative_groups;


namespace epb {
namespace {

constexpr unsigned kFull = 0xffffffffu;
static_assert(kClusterWarps % 8 == 0, "the cluster kernel sums warp counts 8 at a time (16 or 32 warps)");
constexpr int kSmallThreads = 1024;
constexpr int kSmallWarps = kSmallThreads / 32;

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Bits of an expert id in [0, E).
__device__ __forceinline__ int id_bits(int E) { return E > 1 ? 32 - __clz(E - 1) : 0; }

// The lanes in `active` whose v (in [0, 2^bits)) equals this lane's: one
// ballot per bit (a radix match), NB independent ballots issued back to back.
// __match_any_sync did the same in several thousand cycles per call with 32
// warps of a CTA calling it at once. Bits above `bits` are 0 for every lane in
// `active`, so a larger NB gives the same mask.
template <int NB>
__device__ __forceinline__ unsigned warp_peers_n(int v, unsigned active) {
    unsigned m = active;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        const bool one = (v >> b) & 1;
        const unsigned s = __ballot_sync(kFull, one);
        m &= one ? s : ~s;
    }
    return m;
}

__device__ __forceinline__ unsigned warp_peers(int v, int bits, unsigned active) {
    if (bits <= 4) return warp_peers_n<4>(v, active);
    if (bits <= 8) return warp_peers_n<8>(v, active);
    return warp_peers_n<12>(v, active); // kMaxExperts = 2^12
}

// A 32-pair warp step that holds whole tokens (K divides 32, the step starts
// at a multiple of 32): a lane whose id repeats one of a lower lane of the
// same token is dropped (e = -1) and flagged. Returns each kept lane's peers
// among the kept lanes.
__device__ __forceinline__ unsigned whole_token_peers(int &e, int K, int bits, uint32_t &fl) {
    const int lane = threadIdx.x & 31;
    const unsigned peers = warp_peers(e, bits, __ballot_sync(kFull, e >= 0));
    const unsigned tok = K == 32 ? kFull : ((1u << K) - 1u) << (lane & ~(K - 1)); // K is a power of two
    const bool dup = e >= 0 && (peers & tok & lanemask_lt()) != 0;
    if (dup) {
        fl |= EP_FLAG_DUP_EXPERT_ID;
        e = -1;
    }
    return peers & ~__ballot_sync(kFull, dup);
}

// A pair is routed iff its id is in [0, E) and no earlier choice of the same
// token picked that id. -1 is a masked choice (no flag). s_ids starts at a
// token boundary, so the earlier choices of pair p are s_ids[p-k .. p-1].
__device__ __forceinline__ int classify(const int32_t *s_ids, int p, int k, int E, uint32_t &fl) {
    const int e = s_ids[p];
    if (e == -1) return -1;
    if (e < 0 || e >= E) {
        fl |= EP_FLAG_BAD_EXPERT_ID;
        return -1;
    }
    for (int k2 = 1; k2 <= k; ++k2) {
        if (s_ids[p - k2] == e) {
            fl |= EP_FLAG_DUP_EXPERT_ID;
            return -1;
        }
    }
    return e;
}

__device__ __forceinline__ void load_ids(const int32_t *__restrict__ idx, int64_t p0, int np, int32_t *s_ids) {
    for (int i = threadIdx.x; i < np; i += blockDim.x) s_ids[i] = __ldg(idx + p0 + i);
}

__device__ __forceinline__ uint32_t block_or(uint32_t v, uint32_t *s_acc) {
    v = __reduce_or_sync(kFull, v);
    if ((threadIdx.x & 31) == 0 && v) atomicOr(s_acc, v);
    return v;
}

// Exclusive scan of a[0..n) in shared memory by the whole block: calls
// visit(i, prefix of i, a[i]) once for every i, then returns the total.
// s_warp needs 32 ints. Every thread of the block must call it. Two
// barriers: after the warps' totals are stored, every warp scans the 32
// totals itself (instead of one warp scanning them behind a third barrier);
// the second follows the visits.
template <class Visit>
__device__ int block_exscan_visit(const int32_t *a, int n, int32_t *s_warp, Visit visit) {
    const int tid = threadIdx.x, nth = blockDim.x, lane = tid & 31, w = tid >> 5, nw = nth >> 5;
    const int per = (n + nth - 1) / nth;
    const int lo = min(n, tid * per), hi = min(n, lo + per);
    int sum = 0;
    for (int i = lo; i < hi; ++i) sum += a[i];
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) s_warp[w] = incl;
    __syncthreads();
    const int v = lane < nw ? s_warp[lane] : 0;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(kFull, inc, o);
        if (lane >= o) inc += u;
    }
    const int wbase = __shfl_sync(kFull, inc - v, w); // totals of the warps before this one
    const int total = __shfl_sync(kFull, inc, 31);
    int run = wbase + incl - sum;
    for (int i = lo; i < hi; ++i) {
        const int x = a[i];
        visit(i, run, x);
        run += x;
    }
    __syncthreads(); // the visits are complete, and s_warp may be reused
    return total;
}

// The same, leaving the exclusive prefixes in a[].
__device__ int block_exscan(int32_t *a, int n, int32_t *s_warp) {
    return block_exscan_visit(a, n, s_warp, [=](int i, int pre, int) { a[i] = pre; });
}

// One warp walks pairs [lo, hi) of s_ids in (token, k) order, 32 at a time,
// adding the routed pairs of each expert to its own counters my[e].
__device__ __forceinline__ void warp_count(const int32_t *s_ids, int lo, int hi, int K, int E, int32_t *my,
                                           uint32_t &fl) {
    const int lane = threadIdx.x & 31, bits = id_bits(E);
    for (int base = lo; base < hi; base += 32) {
        const int p = base + lane;
        const int e = p < hi ? classify(s_ids, p, p % K, E, fl) : -1;
        const unsigned peers = warp_peers(e, bits, __ballot_sync(kFull, e >= 0));
        if (e >= 0 && (peers & lanemask_lt()) == 0) my[e] += __popc(peers);
        __syncwarp();
    }
}

// Second walk over the same pairs: my[e] now holds the stable index of the
// warp's first pair of expert e; each pair's index j goes through `look`.
template <class Lookup>
__device__ __forceinline__ void warp_assign(const int32_t *s_ids, int lo, int hi, int K, int E, int32_t *my,
                                            int32_t *__restrict__ dest_row, int32_t *__restrict__ src_row,
                                            Lookup look) {
    const int lane = threadIdx.x & 31, bits = id_bits(E);
    uint32_t fl = 0;
    for (int base = lo; base < hi; base += 32) {
        const int p = base + lane;
        const int e = p < hi ? classify(s_ids, p, p % K, E, fl) : -1;
        const unsigned peers = warp_peers(e, bits, __ballot_sync(kFull, e >= 0));
        int dest = -1;
        if (e >= 0) dest = look(e, my[e] + __popc(peers & lanemask_lt()));
        __syncwarp();
        if (e >= 0 && (peers & lanemask_lt()) == 0) my[e] += __popc(peers);
        __syncwarp();
        if (p < hi) dest_row[p] = dest;
        if (dest >= 0 && src_row) src_row[dest] = p;
    }
}

// ---------------------------------------------------------------------------
// layouts (s_cnt holds the per-expert counts of routed pairs)
// ---------------------------------------------------------------------------

// HT: experts in id order; LL: [E][cap] rows, pairs beyond cap dropped.
// Every thread of the CTA calls it; it leaves the kept length and first row
// of every expert in s_len / s_base and returns the number of kept rows.
__device__ int plain_tables(const Dims &d, const int32_t *s_cnt, int32_t *s_len, int32_t *s_base, int32_t *s_warp,
                            uint32_t *s_fl) {
    const int E = d.E, tid = threadIdx.x, nth = blockDim.x;
    const bool ll = d.mode == EP_MODE_LL;
    uint32_t fl = 0;
#pragma unroll 1
    for (int e = tid; e < E; e += nth) {
        const int c = s_cnt[e];
        const int kept = ll ? min(c, d.cap) : c;
        if (ll && c > d.cap) fl |= EP_FLAG_CAPACITY;
        s_len[e] = kept;
        s_base[e] = ll ? e * d.cap : kept;
    }
    block_or(fl, s_fl);
    __syncthreads();
    int total = 0;
    if (!ll) total = block_exscan(s_base, E, s_warp);
    __syncthreads();
    return total;
}

// The plain layout's outputs (one CTA writes them).
__device__ void plain_outputs(const Dims &d, const Workspace &ws, const int32_t *s_len, const int32_t *s_base,
                              int total) {
    const int E = d.E, R = d.R, g = d.g, tid = threadIdx.x, nth = blockDim.x;
    const bool ll = d.mode == EP_MODE_LL;
#pragma unroll 1
    for (int e = tid; e < E; e += nth) {
        ws.len0[e] = s_len[e];
        ws.base0[e] = s_base[e];
        ws.recv_counts[e] = s_len[e];
    }
#pragma unroll 1
    for (int r = tid >> 5; r < R; r += nth >> 5) { // a warp per rank
        int s = 0;
#pragma unroll 1
        for (int i = tid & 31; i < g; i += 32) s += s_len[r * g + i];
        s = __reduce_add_sync(kFull, s);
        if ((tid & 31) == 0) {
            ws.rank_load[r] = s;
            ws.rank_off[r] = ll ? r * g * d.cap : s_base[r * g];
        }
    }
    if (tid == 0) {
        ws.rank_off[R] = ll ? E * d.cap : total;
        *ws.red_count = 0;
    }
}

// A plan's assignment tables as one CTA holds them in shared memory: piece 0
// of expert e is stable indices [0, len0[e]) at rows base0[e] + j; its extra
// pieces are x in [pfirst[e], pfirst[e] + pn[e]), each stable indices
// [xstart[x], xstart[x] + xlen[x]) at rows xdst[x] + (j - xstart[x]).
struct PlanView {
    const int32_t *len0, *base0, *pfirst, *pn, *xstart, *xlen, *xdst;
    __device__ __forceinline__ int dest(int e, int j) const {
        if (j < len0[e]) return base0[e] + j;
        for (int x = pfirst[e], xe = x + pn[e]; x < xe; ++x)
            if (j >= xstart[x] && j < xstart[x] + xlen[x]) return xdst[x] + (j - xstart[x]);
        return -1;
    }
};

// Balanced-replica plan (MoonEP article paras. 3 and 5). The article states
// only the invariants; this is a deterministic greedy:
//  keep     each rank visits its own experts by (count asc, id asc) and keeps
//           rows up to its capacity q or q+1 (q = L/R, first L%R ranks +1);
//  spill    experts with rows left, by (count desc, id asc), fill the ranks
//           with a deficit, visited once in (deficit desc, rank asc) order,
//           each piece taking a new replica slot of the receiving rank
//           (at most S per rank); rows no rank can take stay with the owner
//           and EP_FLAG_PLAN_SLOTS is raised;
//  layout   rank regions in rank order; inside one, own experts in id order
//           then replica slots in slot order.
// Every piece of an expert covers a run of its stable indices; the owner's
// run [0, keep) is piece 0, the others ("extra" pieces) are stored compactly.
//
// Every thread of the CTA calls it. With `publish` the tables go to the
// workspace; in any case the CTA keeps, in its shared memory, what the
// assignment of its own pairs needs (the returned view), valid after the
// function's final barrier.
__device__ PlanView layout_balanced(const Dims &d, const Workspace &ws, const int32_t *s_cnt, int32_t *sm,
                                    int32_t *s_warp, uint32_t *s_fl, bool publish) {
    const int E = d.E, R = d.R, g = d.g, S = d.S, NX = d.nx_max, RS = d.R * d.S;
    const int tid = threadIdx.x, nth = blockDim.x;
    int32_t *s_keep = sm;                   // [E] rows each expert keeps on its owner
    int32_t *s_list = s_keep + E;           // [E] spill flags; then the spilled experts in fill order
    int32_t *s_spill = s_list + E;          // [E] spilled experts in id order; then each one's first receiver
    int32_t *s_spc = s_spill + E;           // [E] their counts; then each one's last receiver; then base0
    int32_t *s_sps = s_spc + E;             // [E] their spilled rows
    int32_t *s_pfirst = s_sps + E;          // [E] first extra piece of each expert (creation order)
    int32_t *s_pn = s_pfirst + E;           // [E] extra pieces of each expert
    int32_t *s_D = s_pn + E;                // [R] deficits
    int32_t *s_used = s_D + R;              // [R] rows each rank keeps of its own experts
    int32_t *s_nrep = s_used + R;           // [R] slots taken (sequential fill)
    int32_t *s_recv = s_nrep + R;           // [R] receivers in visiting order
    int32_t *s_dn = s_recv + R;             // [R] direct pieces per rank
    int32_t *s_fe = s_dn + R;               // [R] expert holding each receiver's first deficit row
    int32_t *s_inner = s_fe + R;            // [R] 1 if that row is not an expert's first spilled row
    int32_t *s_slot_e = s_inner + R;        // [R*S] expert of each replica slot, -1 empty
    // the extra pieces (beyond each expert's own rows) in creation order,
    // which groups them by expert
    int32_t *s_x_start = s_slot_e + RS;     // [NX] first stable index
    int32_t *s_x_len = s_x_start + NX;      // [NX]
    int32_t *s_x_rank = s_x_len + NX;       // [NX] rank holding the piece
    int32_t *s_x_slot = s_x_rank + NX;      // [NX] slot >= 0, -2 owner tail, -3 direct
    int32_t *s_x_aux = s_x_slot + NX;       // [NX] direct: rows before it among the rank's direct rows; then its row
    int32_t *s_A = s_x_aux + NX;            // [E+1] first spilled row of each spilled expert (fill order)
    int32_t *s_B = s_A + E + 1;             // [R+1] first deficit row of each receiver (visiting order)
    // one scan's input, [own rows of each expert | rows of each slot | direct
    // rows of each rank | extra pieces of each expert | expert has replicas |
    // slot is filled]: its prefixes give every offset of the layout
    int32_t *s_seg = s_B + R + 1;
    const int o_slen = E, o_dsum = E + RS, o_x = o_dsum + R, o_rep = o_x + E, o_slot = o_rep + E;
    const int n_seg = o_slot + RS;
    int32_t *q_own = s_seg, *q_slen = s_seg + o_slen, *q_dsum = s_seg + o_dsum, *q_x = s_seg + o_x,
            *q_rep = s_seg + o_rep, *q_slot = s_seg + o_slot;
    __shared__ int s_nrecv, s_seq, s_spill_total;
    __shared__ int s_wsum[32];

    // 0. clear; L = routed pairs
    if (tid == 0) {
        s_nrecv = 0;
        s_seq = 0;
        s_spill_total = 0;
    }
#pragma unroll 1
    for (int i = tid; i < RS; i += nth) s_slot_e[i] = -1;
#pragma unroll 1
    for (int i = tid; i < n_seg; i += nth) s_seg[i] = 0;
#pragma unroll 1
    for (int r = tid; r < R; r += nth) {
        s_used[r] = 0;
        s_nrep[r] = 0;
        s_dn[r] = 0;
    }
    if (d.direct && publish) {
#pragma unroll 1
        for (int i = tid; i < R * E; i += nth) ws.direct_expert[i] = -1;
    }
    int part = 0;
#pragma unroll 1
    for (int e = tid; e < E; e += nth) {
        s_pfirst[e] = 0;
        s_pn[e] = 0;
        part += s_cnt[e];
    }
    part = __reduce_add_sync(kFull, part);
    if ((tid & 31) == 0) s_wsum[tid >> 5] = part;
    __syncthreads();
    const int L = __reduce_add_sync(kFull, (tid & 31) < (nth >> 5) ? s_wsum[tid & 31] : 0);
    const int q = L / R, rem = L % R;
    auto capacity = [&](int r) { return q + (r < rem ? 1 : 0); };

    // 1. keep: rows of the experts visited before e on its rank (sorted order)
    int spilled = 0;
#pragma unroll 1
    for (int e = tid; e < E; e += nth) {
        const int r = e / g, c = s_cnt[e], e0 = r * g;
        int before = 0;
#pragma unroll 8
        for (int i = 0; i < g; ++i) {
            const int c2 = s_cnt[e0 + i];
            before += (c2 < c || (c2 == c && e0 + i < e)) ? c2 : 0;
        }
        const int keep = max(0, min(c, capacity(r) - before));
        s_keep[e] = keep;
        q_own[e] = keep;
        s_list[e] = c > keep ? 1 : 0;
        spilled += c - keep;
        if (keep > 0) atomicAdd(&s_used[r], keep);
    }
    spilled = __reduce_add_sync(kFull, spilled);
    if ((tid & 31) == 0 && spilled) atomicAdd(&s_spill_total, spilled);
    __syncthreads();

    // 2. the spilled experts, compact in id order, with their counts and spilled rows
    const int nsp = block_exscan_visit(s_list, E, s_warp, [&](int e, int pos, int flag) {
        if (flag) {
            s_spill[pos] = e;
            s_spc[pos] = s_cnt[e];
            s_sps[pos] = s_cnt[e] - s_keep[e];
        }
    });

    // 3. fill order: each spilled expert's place by (count desc, id asc) and
    // its first spilled row (the rows of the experts before it); each
    // receiver's place by (deficit desc, rank asc) and its first deficit row
    const int spill_total = s_spill_total;
#pragma unroll 1
    for (int i = tid; i < nsp; i += nth) {
        const int e = s_spill[i], c = s_spc[i];
        int pos = 0, a = 0;
#pragma unroll 8
        for (int i2 = 0; i2 < nsp; ++i2) {
            const int c2 = s_spc[i2], e2 = s_spill[i2], v = s_sps[i2];
            const bool ahead = c2 > c || (c2 == c && e2 < e);
            pos += ahead ? 1 : 0;
            a += ahead ? v : 0;
        }
        s_list[pos] = e;
        s_A[pos] = a;
    }
#pragma unroll 1
    for (int r = tid; r < R; r += nth) {
        const int D = capacity(r) - s_used[r]; // >= 0: no rank keeps more than its capacity
        s_D[r] = D;
        if (D <= 0) continue;
        int pos = 0, b = 0;
#pragma unroll 8
        for (int r2 = 0; r2 < R; ++r2) {
            const int D2 = capacity(r2) - s_used[r2];
            const bool ahead = D2 > 0 && (D2 > D || (D2 == D && r2 < r));
            pos += ahead ? 1 : 0;
            b += ahead ? D2 : 0;
        }
        s_recv[pos] = r;
        s_B[pos] = b;
        atomicAdd(&s_nrecv, 1);
    }
    // the deficits add up to the spilled rows (the capacities add up to L)
    if (tid == 0) s_A[nsp] = spill_total;
    __syncthreads();
    const int nrecv = s_nrecv;
    if (tid == 0) s_B[nrecv] = spill_total; // read after the next barrier

    // the last index i in [0, n) with a[i] <= v (a ascending, a[0] <= v)
    auto last_le = [](const int32_t *a, int n, int v) {
        int lo = 0, hi = n - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (a[mid] <= v) lo = mid; else hi = mid - 1;
        }
        return lo;
    };
    // 4. without a slot running out, the greedy walk pairs the spilled rows
    // (experts in fill order) with the deficit rows (receivers in visiting
    // order) position by position: a piece is the overlap of one expert's
    // spilled rows [A_i, A_i+1) with one receiver's deficit rows [B_q, B_q+1).
    // Receiver q's pieces come from consecutive experts, from the one holding
    // row B_q on, so a piece's slot is its expert's place minus that one's.
    // Per receiver: that expert, whether B_q falls inside its rows, and the
    // check that no receiver needs more than S slots (else, without direct
    // overflow, the walk itself runs below). Per expert: the receivers
    // holding its first and last spilled rows.
#pragma unroll 1
    for (int k = tid; k < nrecv; k += nth) {
        const int b0 = s_B[k], b1 = k + 1 < nrecv ? s_B[k + 1] : spill_total;
        const int fe = last_le(s_A, nsp, b0), le = last_le(s_A, nsp, b1 - 1);
        const int npc = le - fe + 1;
        s_fe[k] = fe;
        s_inner[k] = s_A[fe] < b0 ? 1 : 0;
        if (npc > S) {
            if (!d.direct) {
                s_seq = 1;
            } else { // pieces past the S-th are read directly from the owner
                const int r = s_recv[k];
                s_dn[r] = npc - S;
                q_dsum[r] = b1 - s_A[fe + S];
            }
        }
    }
#pragma unroll 1
    for (int i = tid; i < nsp; i += nth) {
        s_spill[i] = last_le(s_B, nrecv, s_A[i]);
        s_spc[i] = last_le(s_B, nrecv, s_A[i + 1] - 1);
    }
    __syncthreads();

    if (!s_seq) { // uniform: set before the barrier
        // 5. the pieces. Expert i's first piece is i plus the receivers' first
        // rows that fall strictly inside the rows of the experts before it.
#pragma unroll 1
        for (int i = tid; i < nsp; i += nth) {
            const int e = s_list[i], a0 = s_A[i], a1 = s_A[i + 1], qf = s_spill[i], ql = s_spc[i];
            int x = i;
#pragma unroll 8
            for (int k = 1; k <= qf; ++k) x += s_inner[k];
            s_pfirst[e] = x;
            s_pn[e] = ql - qf + 1;
            q_x[e] = ql - qf + 1;
            int rep = 0;
            for (int k = qf; k <= ql; ++k, ++x) {
                const int r = s_recv[k], b0 = s_B[k], b1 = s_B[k + 1];
                const int lo = max(a0, b0), hi = min(a1, b1);
                const int fe = s_fe[k], slot = i - fe;
                s_x_start[x] = s_keep[e] + (lo - a0);
                s_x_len[x] = hi - lo;
                s_x_rank[x] = r;
                if (slot < S) {
                    s_x_slot[x] = slot;
                    s_slot_e[r * S + slot] = e;
                    q_slen[r * S + slot] = hi - lo;
                    q_slot[r * S + slot] = 1;
                    rep = 1;
                } else { // direct piece slot - S of rank r
                    const int first_direct_row = min(b1, s_A[fe + S]);
                    s_x_slot[x] = -3;
                    s_x_aux[x] = lo - first_direct_row;
                    if (publish) {
                        ws.direct_expert[(int64_t)r * E + slot - S] = e;
                        ws.direct_start[(int64_t)r * E + slot - S] = s_keep[e] + (lo - a0);
                        ws.direct_len[(int64_t)r * E + slot - S] = hi - lo;
                    }
                }
            }
            q_rep[e] = rep;
        }
    } else {
        // 5'. the walk itself: one thread, one step per piece (receivers that
        // ran out of deficit or slots never qualify again, so one cursor over
        // them suffices; with direct overflow a receiver out of slots still
        // qualifies and takes the rows as a direct piece). Pieces go to shared
        // memory in creation order.
        if (tid == 0) {
            int p = 0, nx = 0;
            uint32_t fl = 0;
            for (int i = 0; i < nsp; ++i) {
                const int e = s_list[i], owner = e / g;
                int left = s_cnt[e] - s_keep[e], next = s_keep[e], rep = 0;
                s_pfirst[e] = nx;
                while (left > 0) {
                    while (p < nrecv && (s_D[s_recv[p]] == 0 || (!d.direct && s_nrep[s_recv[p]] >= S))) ++p;
                    if (p == nrecv) { // the owner keeps the rest
                        q_own[e] += left;
                        s_x_start[nx] = next;
                        s_x_len[nx] = left;
                        s_x_rank[nx] = owner;
                        s_x_slot[nx] = -2;
                        ++nx;
                        fl |= EP_FLAG_PLAN_SLOTS;
                        break;
                    }
                    const int r = s_recv[p];
                    const int give = min(left, s_D[r]);
                    s_x_start[nx] = next;
                    s_x_len[nx] = give;
                    s_x_rank[nx] = r;
                    if (s_nrep[r] < S) {
                        const int sl = s_nrep[r]++;
                        s_slot_e[r * S + sl] = e;
                        q_slen[r * S + sl] = give;
                        q_slot[r * S + sl] = 1;
                        s_x_slot[nx] = sl;
                        rep = 1;
                    } else { // a direct piece (direct overflow only)
                        const int di = s_dn[r]++;
                        if (publish) {
                            ws.direct_expert[(int64_t)r * E + di] = e;
                            ws.direct_start[(int64_t)r * E + di] = next;
                            ws.direct_len[(int64_t)r * E + di] = give;
                        }
                        s_x_slot[nx] = -3;
                        s_x_aux[nx] = q_dsum[r];
                        q_dsum[r] += give;
                    }
                    ++nx;
                    s_D[r] -= give;
                    left -= give;
                    next += give;
                }
                s_pn[e] = nx - s_pfirst[e];
                q_x[e] = nx - s_pfirst[e];
                q_rep[e] = rep;
            }
            if (fl) atomicOr(s_fl, fl);
        }
    }
    __syncthreads();

    // 6. one scan; then, with P the prefixes (each part's relative to its
    // first element) and v(i) = P(i+1) - P(i) the scanned values:
    //   rank r's region starts at own(r*g) + slots(r*S) + direct(r) and holds
    //   its own experts (offsets own(e) - own(r*g)), then its slots, then its
    //   direct rows
    const int grand = block_exscan(s_seg, n_seg, s_warp);
    const int32_t *P = s_seg;
    auto own_total = [&](int r) { return P[(r + 1) * g] - P[r * g]; };
    auto slot_total = [&](int r) { return P[o_slen + (r + 1) * S] - P[o_slen + r * S]; };
    auto rank_off = [&](int r) { return P[r * g] + (P[o_slen + r * S] - P[o_slen]) + (P[o_dsum + r] - P[o_dsum]); };
    if (publish) {
#pragma unroll 1
        for (int e = tid; e < E; e += nth) // own rows of each own expert
            ws.recv_counts[(int64_t)(e / g) * (g + S) + e % g] = P[e + 1] - P[e];
#pragma unroll 1
        for (int i = tid; i < RS; i += nth) { // rows of each slot; the filled slots, ascending
            ws.recv_counts[(int64_t)(i / S) * (g + S) + g + i % S] = P[o_slen + i + 1] - P[o_slen + i];
            ws.replica_expert[i] = s_slot_e[i];
            if (s_slot_e[i] >= 0) ws.slot_list[P[o_slot + i] - P[o_slot]] = i;
        }
#pragma unroll 1
        for (int r = tid; r < R; r += nth) {
            const int dsum = P[o_dsum + r + 1] - P[o_dsum + r];
            ws.rank_load[r] = own_total(r) + slot_total(r) + dsum;
            ws.rank_off[r] = rank_off(r);
            if (d.direct) ws.direct_n[r] = s_dn[r];
        }
        if (tid == 0) {
            ws.rank_off[R] = P[o_x];
            ws.xoff[E] = P[o_rep] - P[o_x];
            *ws.red_count = P[o_slot] - P[o_rep];
            *ws.slot_count = grand - P[o_slot];
        }
    }
    // piece 0, the extra pieces' rows, and the per-expert replica lists (slots
    // r*S+s in ascending order: each entry's place is the number of the
    // expert's slot pieces with a smaller key)
#pragma unroll 1
    for (int e = tid; e < E; e += nth) {
        const int owner = e / g;
        const int own_base = rank_off(owner) + P[e] - P[owner * g];
        const int xo = P[o_x + e] - P[o_x];
        s_spc[e] = own_base;
        if (publish) {
            ws.base0[e] = own_base;
            ws.len0[e] = s_keep[e];
            ws.xoff[e] = xo;
        }
        const int f = s_pfirst[e], n = s_pn[e];
        int nrep = 0;
        for (int i = 0; i < n; ++i) {
            const int x = f + i, r = s_x_rank[x], sl = s_x_slot[x];
            int dst;
            if (sl == -2) {
                dst = own_base + s_keep[e];
            } else if (sl == -3) { // direct piece: no slot, no gradient to reduce
                dst = rank_off(r) + own_total(r) + slot_total(r) + s_x_aux[x];
            } else {
                dst = rank_off(r) + own_total(r) + P[o_slen + r * S + sl] - P[o_slen + r * S];
                if (publish) {
                    const int key = r * S + sl;
                    int pos = 0;
                    for (int i2 = 0; i2 < n; ++i2) {
                        const int sl2 = s_x_slot[f + i2];
                        if (sl2 >= 0 && s_x_rank[f + i2] * S + sl2 < key) ++pos;
                    }
                    ws.red_list[(int64_t)e * R + pos] = key;
                }
                ++nrep;
            }
            s_x_aux[x] = dst;
            if (publish) {
                ws.xstart[xo + i] = s_x_start[x];
                ws.xlen[xo + i] = s_x_len[x];
                ws.xdst[xo + i] = dst;
            }
        }
        if (publish) {
            ws.red_n[e] = nrep;
            if (nrep > 0) ws.red_experts[P[o_rep + e] - P[o_rep]] = e;
        }
    }
    __syncthreads();
    return PlanView{s_keep, s_spc, s_pfirst, s_pn, s_x_start, s_x_len, s_x_aux};
}

// ---------------------------------------------------------------------------
// 1. per warp tile: validate ids, stable rank of each pair inside the tile,
//    per-expert counts of the tile
// ---------------------------------------------------------------------------
// Each warp owns `wt` consecutive pairs (a warp tile; whole steps of 32).
// packed[p] = e | rank << 16 for a routed pair (rank = earlier pairs of the
// same tile with the same expert), 0xffff otherwise. cnt_tile[tile][e].
__global__ void __launch_bounds__(kRouteThreads) k_route_hist(const int32_t *__restrict__ idx, Dims d,
                                                               Workspace ws) {
    pdl_wait();
    pdl_launch_dependents();
    extern __shared__ int32_t sm[];
    __shared__ uint32_t s_fl;
    const int E = d.E, K = d.K, lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int tile = blockIdx.x * kRouteWarps + w;
    const int row = E + d.wt;           // shared memory per warp
    int32_t *my = sm + w * row;         // [E] counters of this warp's tile
    int32_t *ids = my + E;              // [wt] the tile's expert ids
    if (threadIdx.x == 0) s_fl = 0;
    const int64_t lo = (int64_t)tile * d.wt, hi = min(d.L, lo + d.wt);
    const int n = (int)max((int64_t)0, hi - lo);
    for (int i = lane; i < E; i += 32) my[i] = 0;
    // stage the whole tile first: one memory latency per warp, not per step
    for (int i = lane; i < n; i += 32) ids[i] = __ldg(idx + lo + i);
    __syncthreads();
    uint32_t fl = 0;
    // When K divides 32, every 32-pair step holds whole tokens (tiles start at
    // multiples of 32), so a repeated id is a lane whose (expert, token in
    // step) key matches a lower lane's. Otherwise the earlier choices of the
    // token are compared one by one; k, the lane's choice index, is kept up to
    // date in 32-bit arithmetic.
    const bool whole_tokens = (32 % K) == 0;
    const int step_k = 32 % K, bits = id_bits(E);
    int k = whole_tokens ? 0 : (int)lo % K + lane % K; // pair indices fit 31 bits
    if (k >= K) k -= K;
    for (int base = 0; base < n; base += 32) { // warp-uniform
        const int i = base + lane;
        int e = i < n ? ids[i] : -1;
        if (e != -1 && (e < 0 || e >= E)) {
            fl |= EP_FLAG_BAD_EXPERT_ID;
            e = -1;
        }
        unsigned peers;
        if (whole_tokens) {
            peers = whole_token_peers(e, K, bits, fl);
        } else {
            if (e >= 0) {
                for (int k2 = 1; k2 <= k; ++k2) {
                    const int prev = i - k2 >= 0 ? ids[i - k2] : __ldg(idx + lo + i - k2); // token may start in the previous tile
                    if (prev == e) {
                        fl |= EP_FLAG_DUP_EXPERT_ID;
                        e = -1;
                        break;
                    }
                }
            }
            peers = warp_peers(e, bits, __ballot_sync(kFull, e >= 0));
        }
        const unsigned lower = peers & lanemask_lt();
        int packed = 0xffff;
        if (e >= 0) packed = e | ((my[e] + __popc(lower)) << 16);
        __syncwarp();
        if (e >= 0 && lower == 0) my[e] += __popc(peers);
        __syncwarp();
        if (i < n) ws.packed[lo + i] = packed;
        k += step_k;
        if (k >= K) k -= K;
    }
    block_or(fl, &s_fl);
    __syncthreads();
    // each tile's base among this CTA's tiles, and the CTA's totals
    const int tile0 = blockIdx.x * kRouteWarps;
    const int ntile = min(kRouteWarps, d.ntiles - tile0);
    // the scan kernel's ticket starts every plan at 0, whatever an earlier
    // launch left there (the scan waits for this grid to complete)
    if (d.balanced && blockIdx.x == 0 && threadIdx.x == 0) *ws.ticket = 0ull;
#pragma unroll 1
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
        for (int ww = 0; ww < ntile; ++ww) {
            ws.blk[(int64_t)(tile0 + ww) * E + e] = run;
            run += sm[ww * row + e];
        }
        ws.blk_cta[(int64_t)blockIdx.x * E + e] = run;
    }
    if (threadIdx.x == 0) ws.tile_flags[blockIdx.x] = s_fl;
}

// ---------------------------------------------------------------------------
// 2. per expert: exclusive scan of the tile counts over tiles (lane = expert,
//    warp = a chunk of tiles, so every access is coalesced); with a plan, the
//    CTA that finishes last builds it
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kPlanThreads) k_route_scan(Dims d, Workspace ws) {
    pdl_wait();
    pdl_launch_dependents();
    extern __shared__ int32_t sm[];
    __shared__ int32_t s_warp[33];
    __shared__ int32_t s_part[32][33];
    __shared__ uint32_t s_fl;
    __shared__ int s_last;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, tid = threadIdx.x, nth = blockDim.x;
    const int e = blockIdx.x * 32 + lane;
    const int chunk = (d.nhist + 31) / 32; // rows: one per histogram CTA
    const int t0 = min(d.nhist, w * chunk), t1 = min(d.nhist, t0 + chunk);
    constexpr int B = 16; // loads in flight per thread
    int sum = 0;
    if (e < d.E) {
        for (int t = t0; t < t1; t += B) {
            int v[B];
#pragma unroll
            for (int u = 0; u < B; ++u) v[u] = t + u < t1 ? ws.blk_cta[(int64_t)(t + u) * d.E + e] : 0;
#pragma unroll
            for (int u = 0; u < B; ++u) sum += v[u];
        }
    }
    s_part[w][lane] = sum;
    __syncthreads();
    int run = 0;
    for (int ww = 0; ww < w; ++ww) run += s_part[ww][lane];
    if (e < d.E) {
        for (int t = t0; t < t1; t += B) {
            int v[B];
#pragma unroll
            for (int u = 0; u < B; ++u) v[u] = t + u < t1 ? ws.blk_cta[(int64_t)(t + u) * d.E + e] : 0;
#pragma unroll
            for (int u = 0; u < B; ++u) {
                if (t + u < t1) ws.blk_cta[(int64_t)(t + u) * d.E + e] = run;
                run += v[u];
            }
        }
        if (w == 31) {
            ws.cnt[e] = run;
            if (d.balanced) __threadfence();
        }
    }
    if (!d.balanced) return;
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned long long t = atomicAdd(ws.ticket, 1ull);
        s_last = t + 1 == gridDim.x; // the histogram kernel reset the counter to 0
        s_fl = 0;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    int32_t *s_cnt = sm; // [E]
    uint32_t fl = 0;
    for (int i = tid; i < d.E; i += nth) s_cnt[i] = __ldcg(ws.cnt + i);
    for (int b = tid; b < d.nhist; b += nth) fl |= __ldcg(ws.tile_flags + b);
    block_or(fl, &s_fl);
    __syncthreads();
    layout_balanced(d, ws, s_cnt, sm + d.E, s_warp, &s_fl, true);
    if (tid == 0) *ws.flags = s_fl;
}

// ---------------------------------------------------------------------------
// 3. destination rows: j = tile base + rank in tile, then the layout tables
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kRouteThreads) k_route_assign(Dims d, Workspace ws) {
    pdl_wait();
    pdl_launch_dependents();
    extern __shared__ int32_t sm[];
    __shared__ int32_t s_warp[33];
    __shared__ uint32_t s_fl;
    const int E = d.E, tid = threadIdx.x, nth = blockDim.x;
    int32_t *s_len = sm;         // [E] length of piece 0
    int32_t *s_base = s_len + E; // [E] first row of piece 0
    int32_t *s_cnt = s_base + E; // [E] (plain layouts)
    int32_t *s_xoff = s_cnt + E; // [E+1] extra pieces (plan or world)
    int32_t *s_xs = s_xoff + E + 1;
    int32_t *s_xl = s_xs + d.nx_max;
    int32_t *s_xd = s_xl + d.nx_max;
    int32_t *s_jb = s_xd + d.nx_max; // [E] world: this rank's first stable index per expert
    if (tid == 0) s_fl = 0;
    if (d.balanced || d.world) {
#pragma unroll 1
        for (int i = tid; i < E; i += nth) {
            s_base[i] = ws.base0[i];
            s_len[i] = ws.len0[i];
            if (d.world) s_jb[i] = ws.jbase[i];
        }
        for (int i = tid; i <= E; i += nth) s_xoff[i] = ws.xoff[i];
        const int nx = ws.xoff[E];
        for (int i = tid; i < nx; i += nth) {
            s_xs[i] = ws.xstart[i];
            s_xl[i] = ws.xlen[i];
            s_xd[i] = ws.xdst[i];
        }
        __syncthreads();
    } else {
        for (int i = tid; i < E; i += nth) s_cnt[i] = ws.cnt[i];
        __syncthreads();
        const int total = plain_tables(d, s_cnt, s_len, s_base, s_warp, &s_fl);
        if (blockIdx.x == 0) {
            plain_outputs(d, ws, s_len, s_base, total);
            uint32_t fl = 0;
            for (int b = tid; b < d.nhist; b += nth) fl |= ws.tile_flags[b];
            block_or(fl, &s_fl);
            __syncthreads();
            if (tid == 0) *ws.flags = s_fl;
        }
    }
    // kAssignPer pairs per thread; all loads are issued before any is used
    const int64_t p0 = (int64_t)blockIdx.x * nth * kAssignPer + tid;
    int pk[kAssignPer], jb[kAssignPer];
#pragma unroll
    for (int u = 0; u < kAssignPer; ++u) {
        const int64_t p = p0 + (int64_t)u * nth;
        pk[u] = p < d.L ? ws.packed[p] : 0xffff;
    }
#pragma unroll
    for (int u = 0; u < kAssignPer; ++u) {
        const int64_t p = p0 + (int64_t)u * nth;
        const int e = pk[u] & 0xffff;
        const int64_t tile = p >> d.wt_log2;
        jb[u] = e != 0xffff ? ws.blk_cta[(tile >> kRouteWarpsLog2) * E + e] + ws.blk[tile * E + e] : 0;
    }
#pragma unroll
    for (int u = 0; u < kAssignPer; ++u) {
        const int64_t p = p0 + (int64_t)u * nth;
        if (p >= d.L) continue;
        const int e = pk[u] & 0xffff;
        int dest = -1;
        if (e != 0xffff) {
            const int j = jb[u] + (pk[u] >> 16) + (d.world ? s_jb[e] : 0);
            if (j < s_len[e]) {
                dest = s_base[e] + j;
            } else if (d.balanced || d.world) {
                for (int x = s_xoff[e]; x < s_xoff[e + 1]; ++x)
                    if (j >= s_xs[x] && j < s_xs[x] + s_xl[x]) {
                        dest = s_xd[x] + (j - s_xs[x]);
                        break;
                    }
            }
        }
        ws.dest_row[p] = dest;
        if (dest >= 0 && ws.src_row && !d.world) ws.src_row[dest] = (int32_t)p; // world rows are global
    }
}

// ---------------------------------------------------------------------------
// world plan: the global layout from every rank's counts (one CTA). Every
// rank runs it on the same counts and computes the same tables; jbase holds
// the pairs of expert e on lower ranks, which come first in the expert's
// stable order (source rank, t, k).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kPlanThreads) k_route_world(Dims d, Workspace ws,
                                                               const int32_t *__restrict__ wc, int rank) {
    pdl_wait();
    pdl_launch_dependents();
    extern __shared__ int32_t sm[];
    __shared__ int32_t s_warp[33];
    __shared__ uint32_t s_fl;
    const int E = d.E, R = d.R, tid = threadIdx.x, nth = blockDim.x;
    int32_t *s_cnt = sm;          // [E] the world's counts
    int32_t *s_len = s_cnt + E;   // [E] plain layouts
    int32_t *s_base = s_len + E;  // [E]
    int32_t *s_plan = s_base + E; // the planner's scratch (balanced)
    if (tid == 0) s_fl = 0;
    __syncthreads();
    uint32_t fl = 0; // this rank's id checks, from its histogram CTAs
    for (int b = tid; b < d.nhist; b += nth) fl |= ws.tile_flags[b];
    block_or(fl, &s_fl);
#pragma unroll 1
    for (int e = tid; e < E; e += nth) {
        int all = 0, before = 0;
        for (int r = 0; r < R; ++r) {
            const int v = wc[(int64_t)r * E + e];
            all += v;
            if (r < rank) before += v;
        }
        s_cnt[e] = all;
        ws.cnt[e] = all;
        ws.jbase[e] = before;
        ws.xoff[e] = 0; // plain layouts have no extra pieces; the planner rewrites them
    }
    if (tid == 0) ws.xoff[E] = 0;
    __syncthreads();
    if (d.balanced) {
        layout_balanced(d, ws, s_cnt, s_plan, s_warp, &s_fl, true);
    } else {
        const int total = plain_tables(d, s_cnt, s_len, s_base, s_warp, &s_fl);
        plain_outputs(d, ws, s_len, s_base, total);
    }
    __syncthreads();
    if (tid == 0) *ws.flags = s_fl;
}

// ---------------------------------------------------------------------------
// plain layouts, one cluster: counts, scan, layout and assignment in one launch
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kClusterThreads) k_route_cluster(const int32_t *__restrict__ idx, Dims d,
                                                                    Workspace ws) {
    // first phase of the cluster barrier: this CTA is running. Its wait, just
    // before the first store into another CTA's shared memory, finds every
    // CTA of the cluster started.
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
    pdl_wait();
    pdl_launch_dependents();
    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks(), r = (int)cluster.block_rank();
    extern __shared__ int32_t sm[];
    __shared__ int32_t s_warp[33];
    __shared__ uint32_t s_fl, s_flq[16]; // s_flq[q]: flags of CTA q (pushed by q)
    const int E = d.E, K = d.K, lane = threadIdx.x & 31, w = threadIdx.x >> 5, tid = threadIdx.x;
    const int NW = d.cl_warps; // warps per CTA (blockDim.x / 32)
    const int ppw = d.cl_ppw, ppc = ppw * NW;
    const int64_t c0 = (int64_t)r * ppc;
    const int nc = (int)max((int64_t)0, min((int64_t)ppc, d.L - c0));
    int32_t *s_wc = sm;                     // [warps][E]: per-warp counts, then per-warp bases
    int32_t *s_all = s_wc + NW * E;         // [C][E]: every CTA's totals (pushed by each CTA)
    int32_t *s_cta = s_all + C * E;         // [E]: pairs of each expert in lower-ranked CTAs
    int32_t *s_cnt = s_cta + E;             // [E]: routed pairs per expert (whole batch)
    int32_t *s_len = s_cnt + E;             // [E]: kept rows per expert
    int32_t *s_off = s_len + E;             // [E]: first row of each expert
    int32_t *s_ids = s_off + E;             // [ppc]: this CTA's expert ids
    int32_t *s_pk = s_ids + ppc;            // [ppc]: packed (expert, rank in warp range)
    if (tid == 0) s_fl = 0;
    for (int i = tid; i < NW * E; i += blockDim.x) s_wc[i] = 0;
    for (int i = tid; i < nc; i += blockDim.x) s_ids[i] = __ldg(idx + c0 + i);
    __syncthreads();

    // 1. per warp range: repeat check, rank among the range's pairs of the same expert
    const int lo = w * ppw, hi = min(nc, lo + ppw);
    int32_t *my = s_wc + w * E;
    const bool whole_tokens = (32 % K) == 0; // ranges start at multiples of 32
    const int step_k = 32 % K, bits = id_bits(E);
    int k = whole_tokens ? 0 : ((int)c0 + lo) % K + lane % K; // pair indices fit 31 bits
    if (k >= K) k -= K;
    uint32_t fl = 0;
    for (int base = lo; base < hi; base += 32) { // warp-uniform
        const int i = base + lane;
        int e = i < hi ? s_ids[i] : -1;
        if (e != -1 && (e < 0 || e >= E)) {
            fl |= EP_FLAG_BAD_EXPERT_ID;
            e = -1;
        }
        unsigned peers;
        if (whole_tokens) {
            peers = whole_token_peers(e, K, bits, fl);
        } else {
            if (e >= 0) {
                for (int k2 = 1; k2 <= k; ++k2) {
                    const int prev = i - k2 >= 0 ? s_ids[i - k2] : __ldg(idx + c0 + i - k2);
                    if (prev == e) {
                        fl |= EP_FLAG_DUP_EXPERT_ID;
                        e = -1;
                        break;
                    }
                }
            }
            peers = warp_peers(e, bits, __ballot_sync(kFull, e >= 0));
        }
        const unsigned lower = peers & lanemask_lt();
        if (i < hi) s_pk[i] = e >= 0 ? (e | ((my[e] + __popc(lower)) << 16)) : 0xffff;
        __syncwarp();
        if (e >= 0 && lower == 0) my[e] += __popc(peers);
        __syncwarp();
        k += step_k;
        if (k >= K) k -= K;
    }
    block_or(fl, &s_fl);
    __syncthreads();
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); // every CTA has started
    if (tid < C) *cluster.map_shared_rank(&s_flq[r], tid) = s_fl;
#pragma unroll 1
    for (int e = tid; e < E; e += blockDim.x) { // per-warp bases; the CTA's totals go to every CTA
        int run = 0;
        for (int w0 = 0; w0 < NW; w0 += 8) {
            int v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = s_wc[(w0 + u) * E + e];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                s_wc[(w0 + u) * E + e] = run;
                run += v[u];
            }
        }
#pragma unroll 8
        for (int q = 0; q < C; ++q) cluster.map_shared_rank(s_all, q)[r * E + e] = run;
    }
    // every CTA's stores into this CTA's shared memory are visible after the
    // barrier, and no CTA touches another's shared memory after it
    cluster.sync();

    // 2. totals of the whole batch and of the lower-ranked CTAs, all local now
#pragma unroll 1
    for (int e = tid; e < E; e += blockDim.x) {
        int before = 0, all = 0;
#pragma unroll 8
        for (int q = 0; q < C; ++q) {
            const int v = s_all[q * E + e];
            if (q < r) before += v;
            all += v;
        }
        s_cta[e] = before;
        s_cnt[e] = all;
    }
    if (tid == 0) {
        uint32_t f = 0;
        for (int q = 0; q < C; ++q) f |= s_flq[q];
        s_fl = f;
    }
    __syncthreads();

    if (!d.balanced) {
        // 3. layout (every CTA computes it; CTA 0 publishes it) and assignment
        const int total = plain_tables(d, s_cnt, s_len, s_off, s_warp, &s_fl);
        if (r == 0) {
            plain_outputs(d, ws, s_len, s_off, total);
#pragma unroll 1
            for (int e = tid; e < E; e += blockDim.x) ws.cnt[e] = s_cnt[e];
            __syncthreads();
            if (tid == 0) *ws.flags = s_fl;
        }
#pragma unroll 1
        for (int i = lo + lane; i < hi; i += 32) {
            const int pk = s_pk[i];
            const int e = pk & 0xffff;
            int dest = -1;
            if (e != 0xffff) {
                const int j = s_cta[e] + my[e] + (pk >> 16);
                if (j < s_len[e]) dest = s_off[e] + j;
            }
            ws.dest_row[c0 + i] = dest;
            if (dest >= 0 && ws.src_row) ws.src_row[dest] = (int32_t)(c0 + i);
        }
        return;
    }
    // 3'. balanced plan: every CTA builds it from the totals it now holds, in
    // its own shared memory (CTA 0 also publishes the tables), and assigns its
    // own pairs through its copy
    const PlanView pv = layout_balanced(d, ws, s_cnt, s_pk + ppc, s_warp, &s_fl, r == 0); // scratch: after the pair arrays
    if (r == 0) {
#pragma unroll 1
        for (int e = tid; e < E; e += blockDim.x) ws.cnt[e] = s_cnt[e];
        if (tid == 0) *ws.flags = s_fl; // final: the planner's last barrier follows its last flag
    }
#pragma unroll 1
    for (int i = lo + lane; i < hi; i += 32) {
        const int pk = s_pk[i];
        const int e = pk & 0xffff;
        const int dest = e != 0xffff ? pv.dest(e, s_cta[e] + my[e] + (pk >> 16)) : -1;
        ws.dest_row[c0 + i] = dest;
        if (dest >= 0 && ws.src_row) ws.src_row[dest] = (int32_t)(c0 + i);
    }
}

// ---------------------------------------------------------------------------
// small batches: everything in one CTA (counts, layout or balanced plan,
// assignment), one launch
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kSmallThreads) k_route_small(const int32_t *__restrict__ idx, Dims d,
                                                                Workspace ws) {
    pdl_wait();
    pdl_launch_dependents();
    extern __shared__ int32_t sm[];
    __shared__ int32_t s_warp[33];
    __shared__ uint32_t s_fl;
    const int E = d.E, K = d.K, w = threadIdx.x >> 5, np = (int)d.L;
    int32_t *s_wc = sm;                   // [warps][E]
    int32_t *s_cnt = s_wc + kSmallWarps * E;
    int32_t *s_len = s_cnt + E;           // [E] kept rows (plain) / rows of piece 0 (plan)
    int32_t *s_base = s_len + E;          // [E] first row of the expert / of piece 0
    int32_t *s_ids = s_base + E;          // [L]
    int32_t *s_plan = s_ids + np;         // the planner's scratch (balanced only)
    if (threadIdx.x == 0) s_fl = 0;
    for (int i = threadIdx.x; i < kSmallWarps * E; i += blockDim.x) s_wc[i] = 0;
    load_ids(idx, 0, np, s_ids);
    __syncthreads();
    // each warp owns a contiguous run of pairs; the repeat check reads the
    // earlier choices of a token from s_ids, whichever warp owns them
    const int per_warp = ((np + kSmallWarps - 1) / kSmallWarps + 31) & ~31;
    const int lo = w * per_warp, hi = min(np, lo + per_warp);
    int32_t *my = s_wc + w * E;
    uint32_t fl = 0;
    warp_count(s_ids, lo, hi, K, E, my, fl);
    block_or(fl, &s_fl);
    __syncthreads();
#pragma unroll 1
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
        for (int ww = 0; ww < kSmallWarps; ++ww) {
            const int v = s_wc[ww * E + e];
            s_wc[ww * E + e] = run;
            run += v;
        }
        s_cnt[e] = run;
        ws.cnt[e] = run;
    }
    __syncthreads();
    if (!d.balanced) {
        const int total = plain_tables(d, s_cnt, s_len, s_base, s_warp, &s_fl);
        plain_outputs(d, ws, s_len, s_base, total);
        warp_assign(s_ids, lo, hi, K, E, my, ws.dest_row, ws.src_row,
                    [&](int e, int j) { return j < s_len[e] ? s_base[e] + j : -1; });
    } else {
        // the plan's tables go to the workspace; this CTA assigns its pairs
        // through its own copy in shared memory
        const PlanView pv = layout_balanced(d, ws, s_cnt, s_plan, s_warp, &s_fl, true);
        warp_assign(s_ids, lo, hi, K, E, my, ws.dest_row, ws.src_row, [&](int e, int j) { return pv.dest(e, j); });
    }
    __syncthreads();
    if (threadIdx.x == 0) *ws.flags = s_fl;
}

} // namespace

size_t route_smem_layout(const Dims &d) {
    if (!d.balanced) return 0;
    const size_t E = d.E, R = d.R, RS = (size_t)d.R * d.S, NX = d.nx_max;
    // s_cnt (callers), 7 E-arrays, 7 R-arrays, the slot experts, 5 piece
    // arrays, s_A, s_B, and the scan's input (3 E-parts, 2 slot parts, R)
    return sizeof(int32_t) * (E + 7 * E + 7 * R + RS + 5 * NX + E + 1 + R + 1 + (3 * E + 2 * RS + R));
}

size_t route_smem_assign(const Dims &d) {
    const size_t E = d.E;
    size_t n = 3 * E;
    if (d.balanced || d.world) n += E + 1 + 3 * (size_t)d.nx_max;
    if (d.world) n += E;
    return sizeof(int32_t) * n;
}

size_t route_smem_world(const Dims &d) { return sizeof(int32_t) * 3 * (size_t)d.E + route_smem_layout(d); }

size_t route_smem_hist(const Dims &d) { return sizeof(int32_t) * (size_t)kRouteWarps * (d.E + d.wt); }

size_t route_smem_small(const Dims &d) {
    return sizeof(int32_t) * ((size_t)(kSmallWarps + 3) * d.E + d.L) + route_smem_layout(d);
}

size_t route_smem_cluster(const Dims &d) {
    // with a plan, the planner's scratch follows the pair arrays (every CTA plans)
    return sizeof(int32_t) * ((size_t)(d.cl_warps + 4 + d.cl_size) * d.E + 2 * (size_t)d.cl_ppw * d.cl_warps) +
           route_smem_layout(d);
}

// Can a cluster of d.cl_size CTAs of this kernel be resident at once on this
// device? (Asked once per device and size.)
static bool cluster_fits(const Dims &d) {
    // [device][size 8/16][16/32 warps][smem in 4 KB steps]: 0 unknown, 1 yes, -1 no;
    // threads that race to fill an entry store the same answer
    static std::atomic<signed char> ok[64][2][2][64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    const size_t smem = route_smem_cluster(d);
    const int si = d.cl_size == 16 ? 1 : 0, wi = d.cl_warps == 32 ? 1 : 0, mi = (int)((smem + 4095) / 4096);
    if (mi >= 64) return false;
    signed char known = ok[dev][si][wi][mi].load(std::memory_order_relaxed);
    if (known == 0) {
        cudaFuncSetAttribute(k_route_cluster, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxRouteSmem);
        cudaFuncSetAttribute(k_route_cluster, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(d.cl_size);
        cfg.blockDim = dim3(d.cl_warps * 32);
        cfg.dynamicSmemBytes = (size_t)mi * 4096;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = d.cl_size;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        const cudaError_t e = cudaOccupancyMaxActiveClusters(&n, k_route_cluster, &cfg);
        if (e != cudaSuccess) cudaGetLastError();
        known = (e == cudaSuccess && n >= 1) ? 1 : -1;
        ok[dev][si][wi][mi].store(known, std::memory_order_relaxed);
    }
    return known == 1;
}

bool route_use_cluster(const Dims &d) {
    return d.cl_size > 0 && d.L > (d.balanced ? kSmallMaxPlanPairs : kSmallMaxPairs) && cluster_fits(d);
}

bool route_use_small(const Dims &d) {
    if (d.balanced) return d.L <= kSmallMaxPlanPairs && route_smem_small(d) <= (size_t)kMaxRouteSmem;
    return d.L <= kSmallMaxPairs && d.E <= kSmallMaxExperts;
}

static void set_route_attrs();

cudaError_t launch_plan(const Dims &d, const Workspace &ws, const int32_t *topk_idx, cudaStream_t st) {
    set_route_attrs();
    cudaError_t err;
    if (route_use_cluster(d)) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(d.cl_size);
        cfg.blockDim = dim3(d.cl_warps * 32);
        cfg.dynamicSmemBytes = route_smem_cluster(d);
        cfg.stream = st;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = d.cl_size;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        return cudaLaunchKernelEx(&cfg, k_route_cluster, topk_idx, d, ws);
    }
    if (route_use_small(d))
        return launch_pdl(k_route_small, dim3(1), dim3(kSmallThreads), route_smem_small(d), st, topk_idx, d, ws);
    if (d.L > 0) {
        err = launch_pdl(k_route_hist, dim3(d.nhist), dim3(kRouteThreads), route_smem_hist(d), st, topk_idx, d, ws);
        if (err != cudaSuccess) return err;
    }
    err = launch_pdl(k_route_scan, dim3((d.E + 31) / 32), dim3(kPlanThreads), route_smem_layout(d), st, d, ws);
    if (err != cudaSuccess) return err;
    return launch_pdl(k_route_assign, dim3(d.nassign), dim3(kRouteThreads), route_smem_assign(d), st, d, ws);
}

static void set_route_attrs() {
    // per-device function attributes, set once; the flag is published after them
    static std::atomic<bool> attrs_set[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attrs_set[dev].load(std::memory_order_acquire)) {
        const int max_dyn = kMaxRouteSmem;
        cudaFuncSetAttribute(k_route_hist, cudaFuncAttributeMaxDynamicSharedMemorySize, max_dyn);
        cudaFuncSetAttribute(k_route_assign, cudaFuncAttributeMaxDynamicSharedMemorySize, max_dyn);
        cudaFuncSetAttribute(k_route_scan, cudaFuncAttributeMaxDynamicSharedMemorySize, max_dyn);
        cudaFuncSetAttribute(k_route_small, cudaFuncAttributeMaxDynamicSharedMemorySize, max_dyn);
        cudaFuncSetAttribute(k_route_world, cudaFuncAttributeMaxDynamicSharedMemorySize, max_dyn);
        attrs_set[dev].store(true, std::memory_order_release);
    }
}

// World mode, step 1: the histogram and the per-tile scan of this rank's
// pairs (the three-kernel path's first two kernels, without a plan); the
// per-expert counts are left in ws.cnt.
cudaError_t launch_plan_local_counts(const Dims &d, const Workspace &ws, const int32_t *topk_idx, cudaStream_t st) {
    set_route_attrs();
    Dims dl = d;
    dl.balanced = 0;
    dl.world = 0;
    cudaError_t err;
    if (dl.L > 0) {
        err = launch_pdl(k_route_hist, dim3(dl.nhist), dim3(kRouteThreads), route_smem_hist(dl), st, topk_idx, dl, ws);
        if (err != cudaSuccess) return err;
    }
    return launch_pdl(k_route_scan, dim3((dl.E + 31) / 32), dim3(kPlanThreads), (size_t)0, st, dl, ws);
}

// World mode, step 2: the global layout (one CTA), then each pair's global row.
cudaError_t launch_plan_world(const Dims &d, const Workspace &ws, const int32_t *world_counts, int rank,
                              cudaStream_t st) {
    set_route_attrs();
    Dims dw = d;
    dw.world = 1;
    cudaError_t err =
        launch_pdl(k_route_world, dim3(1), dim3(kPlanThreads), route_smem_world(dw), st, dw, ws, world_counts, rank);
    if (err != cudaSuccess) return err;
    return launch_pdl(k_route_assign, dim3(dw.nassign), dim3(kRouteThreads), route_smem_assign(dw), st, dw, ws);
}

int plan_launches(const Dims &d) {
    return (route_use_cluster(d) || route_use_small(d)) ? 1 : (d.L > 0 ? 3 : 2);
}

} // namespace epb
