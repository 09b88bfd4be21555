/*
 * ep_oracle.c -- CPU oracle for MoE expert-parallel dispatch and combine.
 *
 * TEST INFRASTRUCTURE. Plain, slow, single-threaded C. Only the tests, the
 * smoke check and the benchmark's CPU-baseline / reference leg load this
 * library; the product path never does and shares no code with it (no
 * header, helper, table or constant comes from the CUDA sources).
 *
 * Each routine follows the statement of the problem on these pages:
 *   [NCCL-EP]  the NCCL EP paper page (arXiv 2603.13606): abstract,
 *              Tables II-V, Figs. 2-5.
 *   [MoonEP]   the MoonEP news article (opensourceforu.com): its paragraphs
 *              on the balanced plan, prefetch slots and the reduce buffer
 *              (paragraphs 3-5).
 *   [OFP8]     OCP 8-bit Floating Point Specification, E4M3 format
 *              (the pages name FP8 scales but do not define the format).
 * Where the pages leave a step open, the reading taken is stated beside it.
 *
 * Precision: the pages fix fp32 accumulation in a fixed k order for combine,
 * and fp32 scales of amax/448 for the FP8 cast; the oracle therefore uses
 * float where the method computes in float (compiled with
 * -ffp-contract=off so that no multiply-add is fused unless fmaf() is written).
 *
 * Pins (tests/test_oracle_pins.py): brute-force slot recomputation, layout
 * permutation and load invariants, hand-worked examples under tests/golden/,
 * e4m3 and bf16 rounding against torch's converters, closed forms for the
 * identity and affine experts, fp64 error bounds, adjoint identities.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_FLAG_BAD_EXPERT_ID 1
#define ORC_FLAG_DUP_EXPERT_ID 2
#define ORC_FLAG_CAPACITY 4
#define ORC_FLAG_PLAN_SLOTS 8

/* ------------------------------------------------------------------ */
/* bf16 and e4m3 number formats                                         */
/* ------------------------------------------------------------------ */

float orc_bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a float to the nearest bf16 (8 significant bits), ties to even. */
uint16_t orc_bf16_from_f32(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u) /* NaN: keep it a (quiet) NaN */
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t upper = u >> 16, lower = u & 0xffffu;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u)))
        upper += 1; /* carries into the exponent where the rounding says so */
    return (uint16_t)upper;
}

/* E4M3 [OFP8]: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits.
 * Exponent field 0 holds subnormals m * 2^-9; there is no infinity and the
 * only NaN is S.1111.111, so the largest finite value is 1.75 * 2^8 = 448.
 * Conversion rounds to nearest, ties to even, and saturates finite values
 * beyond 448 to +-448 (the "satfinite" conversion). */
uint8_t orc_e4m3_from_f32(float v) {
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    if (isnan(v)) return (uint8_t)(sign | 0x7f);
    double a = fabs((double)v);
    if (a > 448.0) return (uint8_t)(sign | 0x7e);
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: a multiple of 2^-9; m == 8 is the code of 2^-6 */
        double m = nearbyint(a * 512.0);
        return (uint8_t)(sign | (uint8_t)m);
    }
    int e2;
    (void)frexp(a, &e2); /* a = f * 2^e2 with f in [0.5, 1) */
    int ex = e2 - 1;     /* a = (1 + frac) * 2^ex */
    double m = nearbyint((a / ldexp(1.0, ex) - 1.0) * 8.0);
    if (m == 8.0) {
        ex += 1;
        m = 0.0;
    }
    return (uint8_t)(sign | (uint8_t)(((ex + 7) << 3) | (int)m));
}

float orc_e4m3_to_f32(uint8_t q) {
    int s = q >> 7, e = (q >> 3) & 0xf, m = q & 7;
    double v;
    if (e == 0xf && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return (float)(s ? -v : v);
}

/* Array forms of the converters above, for exhaustive pins. */
void orc_bf16_from_f32_n(const float *v, int64_t n, uint16_t *out) {
    for (int64_t i = 0; i < n; i++) out[i] = orc_bf16_from_f32(v[i]);
}

void orc_e4m3_from_f32_n(const float *v, int64_t n, uint8_t *out) {
    for (int64_t i = 0; i < n; i++) out[i] = orc_e4m3_from_f32(v[i]);
}

/* ------------------------------------------------------------------ */
/* Router: top-K of the gating logits   [Baidu article §2.1, §3.1]     */
/* ------------------------------------------------------------------ */

/* For each token, the K experts with the largest logits (ties: lower id
 * first), in descending order, and their router weights: a softmax over all
 * E logits renormalised over the K chosen ones, which is the softmax of the
 * K chosen logits, w_k = exp(l_k - l_max) / sum_j exp(l_j - l_max), here in
 * double precision, rounded to float once. */
void orc_router_topk(int T, int E, int K, const float *logits, int32_t *idx, float *w) {
    int *taken = (int *)malloc(sizeof(int) * (size_t)E);
    double *ex = (double *)malloc(sizeof(double) * (size_t)K);
    for (int t = 0; t < T; t++) {
        const float *l = logits + (int64_t)t * E;
        for (int e = 0; e < E; e++) taken[e] = 0;
        for (int k = 0; k < K; k++) {
            int best = -1;
            for (int e = 0; e < E; e++) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e; /* strict: the lower id wins a tie */
            }
            taken[best] = 1;
            idx[(int64_t)t * K + k] = best;
        }
        double lmax = l[idx[(int64_t)t * K]], sum = 0.0;
        for (int k = 0; k < K; k++) {
            ex[k] = exp((double)l[idx[(int64_t)t * K + k]] - lmax);
            sum += ex[k];
        }
        for (int k = 0; k < K; k++) w[(int64_t)t * K + k] = (float)(ex[k] / sum);
    }
    free(taken);
    free(ex);
}

/* ------------------------------------------------------------------ */
/* Routing: counts and stable slots   [NCCL-EP Table III; MoonEP para 4] */
/* ------------------------------------------------------------------ */

/* For every (token t, choice k) in row-major order, decide whether the pair
 * is routed and give it its stable index j within its expert: the number of
 * earlier routed pairs (t', k') < (t, k) with the same expert.
 * Reading: id == -1 marks a masked choice (skipped, not an error); any other
 * id outside [0, E) is skipped and flagged; a repeat of an id already chosen
 * by the same token is skipped and flagged. cnt[e] counts routed pairs.
 * j[t*K + k] = -1 for pairs that are not routed. Returns the flag bits. */
int orc_route(int T, int K, int E, const int32_t *idx, int32_t *cnt, int32_t *j) {
    int flags = 0;
    for (int e = 0; e < E; e++) cnt[e] = 0;
    for (int t = 0; t < T; t++) {
        for (int k = 0; k < K; k++) {
            int32_t e = idx[(int64_t)t * K + k];
            int routed = 1;
            if (e == -1) {
                routed = 0;
            } else if (e < 0 || e >= E) {
                routed = 0;
                flags |= ORC_FLAG_BAD_EXPERT_ID;
            } else {
                for (int k2 = 0; k2 < k; k2++)
                    if (idx[(int64_t)t * K + k2] == e) {
                        routed = 0;
                        flags |= ORC_FLAG_DUP_EXPERT_ID;
                    }
            }
            if (routed) {
                j[(int64_t)t * K + k] = cnt[e];
                cnt[e] += 1;
            } else {
                j[(int64_t)t * K + k] = -1;
            }
        }
    }
    return flags;
}

/* HT layout [NCCL-EP Table III "2D with token counts", Fig. 4]: one row per
 * routed pair, rows grouped by expert in ascending id order (so the region of
 * logical rank r = experts r*g .. r*g+g-1 falls out in rank order), each
 * expert's rows in stable (t, k) order: dest = sum_{e' < e} cnt[e'] + j. */
void orc_layout_ht(int T, int K, int E, const int32_t *idx, const int32_t *cnt, const int32_t *j,
                   int32_t *dest_row) {
    (void)E; /* ids were checked against E when the slots were assigned */
    for (int64_t p = 0; p < (int64_t)T * K; p++) {
        if (j[p] < 0) {
            dest_row[p] = -1;
            continue;
        }
        int32_t e = idx[p];
        int64_t off = 0;
        for (int e2 = 0; e2 < e; e2++) off += cnt[e2];
        dest_row[p] = (int32_t)(off + j[p]);
    }
}

/* LL layout [NCCL-EP Table III "3D expert-major", Fig. 3]: buffer
 * [R][E/R][cap][H] = [E][cap][H] since expert e lives on rank e / (E/R) at
 * local index e % (E/R). Row of (t, k) = e * cap + j while j < cap; pairs
 * past the capacity are dropped and flagged. */
int orc_layout_ll(int T, int K, int cap, const int32_t *idx, const int32_t *j, int32_t *dest_row) {
    int flags = 0;
    for (int64_t p = 0; p < (int64_t)T * K; p++) {
        if (j[p] < 0) {
            dest_row[p] = -1;
        } else if (j[p] >= cap) {
            dest_row[p] = -1;
            flags |= ORC_FLAG_CAPACITY;
        } else {
            dest_row[p] = (int32_t)((int64_t)idx[p] * cap + j[p]);
        }
    }
    return flags;
}

/* ------------------------------------------------------------------ */
/* Balanced-replica plan   [MoonEP paras 3 and 5]                       */
/* ------------------------------------------------------------------ */
/*
 * The article states the invariants only: every rank receives a predictable
 * workload whatever the routing skew, hot experts are replicated online from
 * the current router output, and training reserves at most E/R prefetch
 * slots per rank. It gives no algorithm; this deterministic greedy is the
 * reading taken (L = sum cnt, q = L / R, first L mod R ranks take q + 1):
 *
 *  1. keep:     each rank visits its own experts by (cnt ascending, id
 *               ascending) and keeps keep_e = min(cnt_e, cap_r - used) rows,
 *               so cold experts stay home and the hottest spill.
 *  2. deficit:  D_r = cap_r - sum of keep over the rank's experts.
 *  3. spill:    experts with cnt_e - keep_e > 0, by (cnt descending, id
 *               ascending).
 *  4. receivers: ranks with D_r > 0, ordered once by (D descending, rank
 *               ascending).
 *  5. fill:     for each spilled expert, while rows are left, take the first
 *               receiver in that order with D > 0 and fewer than S replica
 *               slots; give it min(left, D) rows as its next slot.
 *               If none qualifies the rows stay with the owner (appended
 *               after its kept rows) and PLAN_SLOTS is flagged.
 *  6. rows:     the owner holds stable indices [0, keep_e), the replica
 *               pieces follow in creation order, then any leftover tail.
 *  7. layout:   rank r's region starts at the sum of the loads of ranks < r;
 *               inside it come its own experts in id order, then its replica
 *               slots in slot order.
 *
 * Outputs: keep[E], tail_start[E] (-1 if none), tail_len[E],
 * replica_expert[R*S] (-1 = empty), slot_start[R*S] (first stable index the
 * slot holds), slot_len[R*S], rank_load[R], rank_off[R+1].
 */
/* Inference variant [MoonEP para 5: at inference a rank keeps only a few
 * prefetch slots and rows past them read the owner's weights in place],
 * reading taken: with
 * `direct` set, step 5 no longer skips a receiver that has a deficit but no
 * free slot; the piece goes to it as a *direct* piece, whose rows are computed
 * with the owner's weights read in place, so every spilled row is placed and
 * loads are always exact. Direct pieces of rank r (at most one per expert)
 * are listed in creation order in direct_expert / direct_start / direct_len
 * [r*E + i], i < direct_n[r]; in r's region they follow its replica slots. */
static int plan_core(int E, int R, int S, int direct, const int32_t *cnt, int32_t *keep, int32_t *tail_start,
                     int32_t *tail_len, int32_t *replica_expert, int32_t *slot_start, int32_t *slot_len,
                     int32_t *direct_n, int32_t *direct_expert, int32_t *direct_start, int32_t *direct_len,
                     int32_t *rank_load, int32_t *rank_off) {
    int g = E / R, flags = 0;
    int64_t L = 0;
    for (int e = 0; e < E; e++) L += cnt[e];
    int64_t q = L / R, rem = L % R;
    int *order = (int *)malloc(sizeof(int) * (size_t)(E > R ? E : R));
    int64_t *D = (int64_t *)malloc(sizeof(int64_t) * (size_t)R);
    int *nrep = (int *)calloc((size_t)R, sizeof(int));

    for (int i = 0; i < R * S; i++) {
        replica_expert[i] = -1;
        slot_start[i] = 0;
        slot_len[i] = 0;
    }
    if (direct) {
        for (int r = 0; r < R; r++) direct_n[r] = 0;
        for (int i = 0; i < R * E; i++) {
            direct_expert[i] = -1;
            direct_start[i] = 0;
            direct_len[i] = 0;
        }
    }
    /* 1-2: keep and deficit per rank */
    for (int r = 0; r < R; r++) {
        int64_t cap = q + (r < rem ? 1 : 0), used = 0;
        for (int i = 0; i < g; i++) order[i] = r * g + i;
        for (int a = 1; a < g; a++) { /* insertion sort by (cnt asc, id asc) */
            int v = order[a], b = a - 1;
            while (b >= 0 && (cnt[order[b]] > cnt[v] || (cnt[order[b]] == cnt[v] && order[b] > v))) {
                order[b + 1] = order[b];
                b--;
            }
            order[b + 1] = v;
        }
        for (int i = 0; i < g; i++) {
            int e = order[i];
            int64_t k = cap - used;
            if (k > cnt[e]) k = cnt[e];
            keep[e] = (int32_t)k;
            used += k;
        }
        D[r] = cap - used;
    }
    /* 3: spilled experts by (cnt desc, id asc) */
    int nsp = 0;
    for (int e = 0; e < E; e++) {
        tail_start[e] = -1;
        tail_len[e] = 0;
        if (cnt[e] - keep[e] > 0) order[nsp++] = e;
    }
    for (int a = 1; a < nsp; a++) {
        int v = order[a], b = a - 1;
        while (b >= 0 && (cnt[order[b]] < cnt[v] || (cnt[order[b]] == cnt[v] && order[b] > v))) {
            order[b + 1] = order[b];
            b--;
        }
        order[b + 1] = v;
    }
    /* 4: receivers by (D desc, rank asc), fixed once */
    int *recv = (int *)malloc(sizeof(int) * (size_t)R);
    int nrecv = 0;
    for (int r = 0; r < R; r++)
        if (D[r] > 0) recv[nrecv++] = r;
    for (int a = 1; a < nrecv; a++) {
        int v = recv[a], b = a - 1;
        while (b >= 0 && (D[recv[b]] < D[v] || (D[recv[b]] == D[v] && recv[b] > v))) {
            recv[b + 1] = recv[b];
            b--;
        }
        recv[b + 1] = v;
    }
    /* 5-6: fill */
    for (int i = 0; i < nsp; i++) {
        int e = order[i];
        int64_t left = cnt[e] - keep[e], next = keep[e];
        while (left > 0) {
            int chosen = -1;
            for (int a = 0; a < nrecv; a++) {
                int r = recv[a];
                if (D[r] > 0 && (nrep[r] < S || direct)) {
                    chosen = r;
                    break;
                }
            }
            if (chosen < 0) {
                tail_start[e] = (int32_t)next;
                tail_len[e] = (int32_t)left;
                flags |= ORC_FLAG_PLAN_SLOTS;
                break;
            }
            int64_t give = left < D[chosen] ? left : D[chosen];
            if (nrep[chosen] < S) {
                int s = nrep[chosen]++;
                replica_expert[chosen * S + s] = e;
                slot_start[chosen * S + s] = (int32_t)next;
                slot_len[chosen * S + s] = (int32_t)give;
            } else { /* a direct piece (only reachable with `direct`) */
                int i = direct_n[chosen]++;
                direct_expert[chosen * E + i] = e;
                direct_start[chosen * E + i] = (int32_t)next;
                direct_len[chosen * E + i] = (int32_t)give;
            }
            D[chosen] -= give;
            left -= give;
            next += give;
        }
    }
    /* 7: loads and rank offsets */
    rank_off[0] = 0;
    for (int r = 0; r < R; r++) {
        int64_t load = 0;
        for (int i = 0; i < g; i++) load += keep[r * g + i] + tail_len[r * g + i];
        for (int s = 0; s < S; s++) load += slot_len[r * S + s];
        if (direct)
            for (int i = 0; i < direct_n[r]; i++) load += direct_len[r * E + i];
        rank_load[r] = (int32_t)load;
        rank_off[r + 1] = (int32_t)(rank_off[r] + load);
    }
    free(order);
    free(D);
    free(nrep);
    free(recv);
    return flags;
}

int orc_plan_balanced(int E, int R, int S, const int32_t *cnt, int32_t *keep, int32_t *tail_start,
                      int32_t *tail_len, int32_t *replica_expert, int32_t *slot_start, int32_t *slot_len,
                      int32_t *rank_load, int32_t *rank_off) {
    return plan_core(E, R, S, 0, cnt, keep, tail_start, tail_len, replica_expert, slot_start, slot_len, NULL,
                     NULL, NULL, NULL, rank_load, rank_off);
}

int orc_plan_direct(int E, int R, int S, const int32_t *cnt, int32_t *keep, int32_t *tail_start, int32_t *tail_len,
                    int32_t *replica_expert, int32_t *slot_start, int32_t *slot_len, int32_t *direct_n,
                    int32_t *direct_expert, int32_t *direct_start, int32_t *direct_len, int32_t *rank_load,
                    int32_t *rank_off) {
    return plan_core(E, R, S, 1, cnt, keep, tail_start, tail_len, replica_expert, slot_start, slot_len, direct_n,
                     direct_expert, direct_start, direct_len, rank_load, rank_off);
}

/* Destination row of every routed pair under a balanced plan (step 6-7). */
static void layout_core(int T, int K, int E, int R, int S, const int32_t *idx, const int32_t *j,
                        const int32_t *keep, const int32_t *tail_start, const int32_t *tail_len,
                        const int32_t *replica_expert, const int32_t *slot_start, const int32_t *slot_len,
                        const int32_t *direct_n, const int32_t *direct_expert, const int32_t *direct_start,
                        const int32_t *direct_len, const int32_t *rank_off, int32_t *dest_row) {
    int g = E / R;
    for (int64_t p = 0; p < (int64_t)T * K; p++) {
        dest_row[p] = -1;
        if (j[p] < 0) continue;
        int e = idx[p], owner = e / g;
        int64_t own_off = 0; /* own experts of the owner in id order */
        for (int e2 = owner * g; e2 < e; e2++) own_off += keep[e2] + tail_len[e2];
        if (j[p] < keep[e]) {
            dest_row[p] = (int32_t)(rank_off[owner] + own_off + j[p]);
            continue;
        }
        if (tail_start[e] >= 0 && j[p] >= tail_start[e] && j[p] < tail_start[e] + tail_len[e]) {
            dest_row[p] = (int32_t)(rank_off[owner] + own_off + keep[e] + (j[p] - tail_start[e]));
            continue;
        }
        for (int r = 0; r < R; r++) {
            for (int s = 0; s < S; s++) {
                int sl = r * S + s;
                if (replica_expert[sl] != e) continue;
                if (j[p] < slot_start[sl] || j[p] >= slot_start[sl] + slot_len[sl]) continue;
                int64_t off = rank_off[r];
                for (int e2 = r * g; e2 < r * g + g; e2++) off += keep[e2] + tail_len[e2];
                for (int s2 = 0; s2 < s; s2++) off += slot_len[r * S + s2];
                dest_row[p] = (int32_t)(off + (j[p] - slot_start[sl]));
            }
        }
        if (!direct_n) continue;
        for (int r = 0; r < R; r++) { /* direct pieces follow the rank's slots */
            for (int i = 0; i < direct_n[r]; i++) {
                if (direct_expert[r * E + i] != e) continue;
                if (j[p] < direct_start[r * E + i] || j[p] >= direct_start[r * E + i] + direct_len[r * E + i])
                    continue;
                int64_t off = rank_off[r];
                for (int e2 = r * g; e2 < r * g + g; e2++) off += keep[e2] + tail_len[e2];
                for (int s2 = 0; s2 < S; s2++) off += slot_len[r * S + s2];
                for (int i2 = 0; i2 < i; i2++) off += direct_len[r * E + i2];
                dest_row[p] = (int32_t)(off + (j[p] - direct_start[r * E + i]));
            }
        }
    }
}

void orc_layout_balanced(int T, int K, int E, int R, int S, const int32_t *idx, const int32_t *j,
                         const int32_t *keep, const int32_t *tail_start, const int32_t *tail_len,
                         const int32_t *replica_expert, const int32_t *slot_start, const int32_t *slot_len,
                         const int32_t *rank_off, int32_t *dest_row) {
    layout_core(T, K, E, R, S, idx, j, keep, tail_start, tail_len, replica_expert, slot_start, slot_len, NULL, NULL,
                NULL, NULL, rank_off, dest_row);
}

void orc_layout_direct(int T, int K, int E, int R, int S, const int32_t *idx, const int32_t *j, const int32_t *keep,
                       const int32_t *tail_start, const int32_t *tail_len, const int32_t *replica_expert,
                       const int32_t *slot_start, const int32_t *slot_len, const int32_t *direct_n,
                       const int32_t *direct_expert, const int32_t *direct_start, const int32_t *direct_len,
                       const int32_t *rank_off, int32_t *dest_row) {
    layout_core(T, K, E, R, S, idx, j, keep, tail_start, tail_len, replica_expert, slot_start, slot_len, direct_n,
                direct_expert, direct_start, direct_len, rank_off, dest_row);
}

/* ------------------------------------------------------------------ */
/* Dispatch   [NCCL-EP Table V dispatch call; Table IV tensor roles]   */
/* ------------------------------------------------------------------ */

/* FP8 cast of one token row [NCCL-EP Table IV "FP8 quantization scales"],
 * per 128-element block b: amax = max |x|, s = amax / 448 (fp32 division),
 * q_i = e4m3(x_i / s) (fp32 division, then RNE with saturation). Reading for
 * an all-zero block: s = 0 and every code is +0. */
static void quant_row(const uint16_t *x, int H, uint8_t *q, float *scales) {
    for (int b = 0; b < H / 128; b++) {
        float amax = 0.0f;
        for (int i = 0; i < 128; i++) {
            float a = fabsf(orc_bf16_to_f32(x[b * 128 + i]));
            if (a > amax) amax = a;
        }
        float s = amax / 448.0f;
        scales[b] = s;
        for (int i = 0; i < 128; i++) {
            if (amax == 0.0f)
                q[b * 128 + i] = 0;
            else
                q[b * 128 + i] = orc_e4m3_from_f32(orc_bf16_to_f32(x[b * 128 + i]) / s);
        }
    }
}

/* recv[dest_row[t,k]] = x[t] (bf16 rows), or its FP8 cast with per-block
 * scales recv_scales[dest_row[t,k]][H/128]; recv_w[row] = w[t,k] and
 * recv_expert[row] = idx[t,k] for every routed pair. Rows that no pair
 * targets are left untouched. recv_w / recv_expert may be NULL. */
void orc_dispatch(int T, int K, int H, int fp8, const uint16_t *x, const int32_t *idx, const float *w,
                  const int32_t *dest_row, void *recv, float *recv_scales, float *recv_w,
                  int32_t *recv_expert) {
    uint8_t *qrow = (uint8_t *)malloc((size_t)H);
    float *srow = (float *)malloc(sizeof(float) * (size_t)(H / 128 + 1));
    for (int t = 0; t < T; t++) {
        const uint16_t *xr = x + (int64_t)t * H;
        if (fp8) quant_row(xr, H, qrow, srow);
        for (int k = 0; k < K; k++) {
            int64_t p = (int64_t)t * K + k;
            int32_t row = dest_row[p];
            if (row < 0) continue;
            if (fp8) {
                memcpy((uint8_t *)recv + (int64_t)row * H, qrow, (size_t)H);
                memcpy(recv_scales + (int64_t)row * (H / 128), srow, sizeof(float) * (size_t)(H / 128));
            } else {
                memcpy((uint16_t *)recv + (int64_t)row * H, xr, sizeof(uint16_t) * (size_t)H);
            }
            if (recv_w) recv_w[row] = w[p];
            if (recv_expert) recv_expert[row] = idx[p];
        }
    }
    free(qrow);
    free(srow);
}

/* ------------------------------------------------------------------ */
/* Combine   [NCCL-EP Table II combine row, Table III "Reduction"]     */
/* ------------------------------------------------------------------ */

/* out[t] = bf16( fold over k = 0..K-1 of acc = fmaf(w[t,k], y[dest_row[t,k]], acc) ),
 * acc starting at +0.0f, pairs that are not routed skipped. With w == NULL
 * the fold is a plain fp32 sum acc = acc + y (the dispatch-gradient combine
 * of the backward pass, Fig. 5). */
void orc_combine(int T, int K, int H, const uint16_t *y, const float *w, const int32_t *dest_row,
                 uint16_t *out) {
    for (int t = 0; t < T; t++) {
        for (int i = 0; i < H; i++) {
            float acc = 0.0f;
            for (int k = 0; k < K; k++) {
                int32_t row = dest_row[(int64_t)t * K + k];
                if (row < 0) continue;
                float v = orc_bf16_to_f32(y[(int64_t)row * H + i]);
                if (w)
                    acc = fmaf(w[(int64_t)t * K + k], v, acc);
                else
                    acc = acc + v;
            }
            out[(int64_t)t * H + i] = orc_bf16_from_f32(acc);
        }
    }
}

/* Backward of combine [NCCL-EP Fig. 5, routing state reused]: the gradient
 * of out[t] flows to every routed row, scaled by its router weight:
 * gy[dest_row[t,k]] = bf16(w[t,k] * float(g[t])) with the product rounded
 * to fp32 and then to bf16 (reading: one fp32 multiply, one bf16 rounding). */
void orc_combine_backward(int T, int K, int H, const uint16_t *g, const float *w, const int32_t *dest_row,
                          uint16_t *gy) {
    for (int t = 0; t < T; t++) {
        for (int k = 0; k < K; k++) {
            int32_t row = dest_row[(int64_t)t * K + k];
            if (row < 0) continue;
            float wk = w[(int64_t)t * K + k];
            for (int i = 0; i < H; i++) {
                float prod = wk * orc_bf16_to_f32(g[(int64_t)t * H + i]);
                gy[(int64_t)row * H + i] = orc_bf16_from_f32(prod);
            }
        }
    }
}

/* ------------------------------------------------------------------ */
/* Replica weight prefetch   [MoonEP paras 3 and 5, prefetch slots]     */
/* ------------------------------------------------------------------ */

/* Every replica slot (r, s) that the plan fills with expert e receives a copy
 * of e's weights: slots[r*S+s] = weights[e] (bytes_per_expert bytes each).
 * Empty slots (replica_expert = -1) are left as they are. */
void orc_prefetch(int R, int S, int64_t bytes_per_expert, const int32_t *replica_expert, const void *weights,
                  void *slots) {
    for (int sl = 0; sl < R * S; sl++) {
        int e = replica_expert[sl];
        if (e < 0) continue;
        memcpy((char *)slots + (int64_t)sl * bytes_per_expert, (const char *)weights + (int64_t)e * bytes_per_expert,
               (size_t)bytes_per_expert);
    }
}

/* ------------------------------------------------------------------ */
/* Replica-gradient reduce   [MoonEP para 5, backward reduce buffer]    */
/* ------------------------------------------------------------------ */

/* owner[e] = owner[e] + sum over slots (r, s) in ascending (r, s) order with
 * replica_expert[r*S+s] == e of rep[r][s], element-wise, fp32 adds in that
 * order. rep is [R*S][G] fp32, owner is [E][G] fp32. Experts with no replica
 * are left untouched. */
void orc_replica_reduce(int E, int R, int S, int64_t G, const int32_t *replica_expert, const float *rep,
                        float *owner) {
    int *list = (int *)malloc(sizeof(int) * (size_t)(R * S + 1));
    for (int e = 0; e < E; e++) {
        int n = 0;
        for (int sl = 0; sl < R * S; sl++)
            if (replica_expert[sl] == e) list[n++] = sl;
        if (n == 0) continue;
        for (int64_t i = 0; i < G; i++) {
            float acc = owner[(int64_t)e * G + i];
            for (int a = 0; a < n; a++) acc = acc + rep[(int64_t)list[a] * G + i];
            owner[(int64_t)e * G + i] = acc;
        }
    }
    free(list);
}
