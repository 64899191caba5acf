/*
 * CPU oracle for the UltraEP balancer's per-layer, per-microbatch hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the tests, the smoke check and the timed CPU baseline
 * of the benchmark use it.  It shares no code, header, table or constant with
 * the CUDA library: every step below is a plain, single-threaded restatement
 * of what the step computes, written for a reader to check by eye.
 *
 * Sources.  "How dots-infra/ultraep works" (gitdiagram summary, component
 * list "GPU operations" and its "Connections") names the five steps: load
 * computation, placement planning, routing expansion, replica weight sync and
 * replica gradient reduction.  The UltraEP news summary ("Comment fonctionne
 * l'équilibrage en 300 microsecondes") calls the planner a quota-driven,
 * exact-load scheduler that runs right after gating.  The exact plan rule
 * taken here: Q = ceil(sum of loads / N); each expert's home rank takes
 * min(load, Q - current); overflow goes greedily, largest overflow first, to
 * the rank with the most spare capacity (ties to the lowest rank id), with at
 * most R replicas per rank; the j-th occurrence of expert e in token-major
 * (t, k) order goes to the replica whose cumulative quota covers j.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - expert e lives on home rank e / H in local slot e % H, H = E / N;
 *     physical slot id = r * (H + R) + s, redundant local slots s in [H, H+R);
 *   - the home pass visits experts in increasing id;
 *   - overflow order is fixed once after the home pass: overflow descending,
 *     ties to the lower expert id; each expert is placed fully before the next;
 *   - a rank is eligible while it has a free redundant slot and spare > 0;
 *   - if no rank is eligible ("slots run out") the remaining overflow stays on
 *     the expert's home slot, which then exceeds Q, and flag bit 0 is set;
 *   - replica order for the cumulative quotas: home slot first, then the
 *     redundant slots in allocation order; j is 0-based;
 *   - the per-rank histogram partitions tokens by source rank t / (T / N);
 *   - ids outside [0, E) are not counted and are rerouted to -1;
 *   - gradient reduction adds replica gradients into the fp32 master in
 *     replica order, widening bf16 exactly, one fp32 round-to-nearest add each.
 *
 * Every function returns 0 on success and a negative code on a violated
 * precondition or a broken internal invariant.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_BAD_ARG (-1)
#define ORC_INVARIANT (-2)

/* ---- step 1: load computation --------------------------------------------
 * counts[r][e] = number of (t, k) with t in rank r's tokens and ids[t][k] = e.
 * bad[r] = number of ids of rank r's tokens outside [0, E).
 */
int ue_oracle_load(const int32_t *ids, int64_t T, int K, int E, int N,
                   int32_t *counts, int32_t *bad)
{
    if (T < 0 || K < 1 || E < 1 || N < 1 || T % N != 0) return ORC_BAD_ARG;
    int64_t tokens_per_rank = T / N;
    memset(counts, 0, sizeof(int32_t) * (size_t)N * (size_t)E);
    if (bad) memset(bad, 0, sizeof(int32_t) * (size_t)N);
    for (int64_t t = 0; t < T; ++t) {
        int64_t r = t / tokens_per_rank;
        for (int k = 0; k < K; ++k) {
            int32_t e = ids[t * K + k];
            if (e < 0 || e >= E) {
                if (bad) bad[r] += 1;
                continue;
            }
            counts[r * E + e] += 1;
        }
    }
    return ORC_OK;
}

/* load[e] = sum over ranks of counts[r][e];
 * rank_off[r][e] = sum over ranks r' < r of counts[r'][e], i.e. how many
 * occurrences of e precede rank r's first token in token-major order. */
int ue_oracle_expert_load(const int32_t *counts, int N, int E,
                          int32_t *load, int32_t *rank_off)
{
    if (N < 1 || E < 1) return ORC_BAD_ARG;
    for (int e = 0; e < E; ++e) {
        int64_t run = 0;
        for (int r = 0; r < N; ++r) {
            if (rank_off) rank_off[(int64_t)r * E + e] = (int32_t)run;
            run += counts[(int64_t)r * E + e];
        }
        if (run > INT32_MAX) return ORC_BAD_ARG;
        load[e] = (int32_t)run;
    }
    return ORC_OK;
}

/* ---- step 2: quota-driven placement planning -----------------------------
 * Outputs (all caller-allocated):
 *   slot_expert[S], slot_quota[S]  S = N*(H+R); empty slots: -1 / 0
 *   rep_off[E+1]                   replicas of e are entries rep_off[e] .. rep_off[e+1]-1
 *   rep_slot[E+N*R], rep_cum[E+N*R] slot of each replica, exclusive prefix of quotas
 *                                   (entries past rep_off[E] are set to -1)
 *   rep_experts[E]                 experts holding >= 1 redundant replica, increasing id (-1 tail)
 *   rank_load_before[N], rank_load_after[N]
 *   info[8] = { Q, L, flags (bit 0: slots ran out), M = #rep_experts,
 *               filled redundant slots, max rank load before, max after, 0 }
 */
typedef struct { int32_t ovf; int32_t e; } orc_ovf;

static int orc_ovf_cmp(const void *a, const void *b)
{
    const orc_ovf *x = (const orc_ovf *)a, *y = (const orc_ovf *)b;
    if (x->ovf != y->ovf) return x->ovf > y->ovf ? -1 : 1;   /* larger overflow first */
    return x->e < y->e ? -1 : (x->e > y->e ? 1 : 0);         /* tie: lower expert id */
}

/* Plan variants (bit flags; 0 = the stated rule):
 *   ORC_REQUEUE  the overflow is a priority queue: after every chunk the expert
 *                with the largest remaining overflow (ties: lower id) is placed
 *                next, instead of placing each expert fully in the order fixed
 *                after the home pass;
 *   ORC_SPREAD   when slots run out, each stuck expert's remainder (in the
 *                order the experts are visited) is spread over its replicas one
 *                token at a time, each token to the replica whose rank has the
 *                lowest load (ties: the earlier replica, home first), instead of
 *                staying on the home slot.
 */
#define ORC_REQUEUE 1
#define ORC_SPREAD 2

int ue_oracle_plan_ex(int E, int N, int R, const int32_t *load, int variant,
                      int32_t *slot_expert, int32_t *slot_quota,
                      int32_t *rep_off, int32_t *rep_slot, int32_t *rep_cum,
                      int32_t *rep_experts,
                      int32_t *rank_load_before, int32_t *rank_load_after,
                      int32_t *info)
{
    if (E < 1 || N < 1 || R < 0 || E % N != 0 || variant < 0 || variant > 3) return ORC_BAD_ARG;
    const int H = E / N, HR = H + R, S = N * HR, NR = N * R;
    int64_t L = 0;
    for (int e = 0; e < E; ++e) {
        if (load[e] < 0) return ORC_BAD_ARG;
        L += load[e];
    }
    if (L > INT32_MAX) return ORC_BAD_ARG;
    const int64_t Q = (L == 0) ? 0 : (L + N - 1) / N;        /* Q = ceil(L / N) */

    int64_t *cur = calloc((size_t)N, sizeof(int64_t));        /* tokens taken by rank r */
    int32_t *used = calloc((size_t)N, sizeof(int32_t));       /* redundant slots used on r */
    int64_t *home_quota = calloc((size_t)E, sizeof(int64_t));
    int64_t *ovf = calloc((size_t)E, sizeof(int64_t));
    orc_ovf *order = calloc((size_t)E, sizeof(orc_ovf));
    int32_t *asg_e = calloc((size_t)NR + 1, sizeof(int32_t)); /* assignments, allocation order */
    int32_t *asg_s = calloc((size_t)NR + 1, sizeof(int32_t));
    int64_t *asg_c = calloc((size_t)NR + 1, sizeof(int64_t));
    int64_t *rem_e = calloc((size_t)E, sizeof(int64_t));      /* remaining overflow (variants) */
    int32_t *stuck = calloc((size_t)E, sizeof(int32_t));      /* experts left with a remainder, in visit order */
    int rc = ORC_OK;
    if (!cur || !used || !home_quota || !ovf || !order || !asg_e || !asg_s || !asg_c || !rem_e || !stuck) {
        rc = ORC_BAD_ARG;
        goto done;
    }
    int flags = 0, n_asg = 0;

    /* Home pass: experts in increasing id; the home rank takes min(load, Q - cur). */
    for (int e = 0; e < E; ++e) {
        int h = e / H;
        int64_t take = load[e] < Q - cur[h] ? load[e] : Q - cur[h];
        cur[h] += take;
        home_quota[e] = take;
        ovf[e] = load[e] - take;
    }

    /* Overflow order, fixed once: largest overflow first, ties to lower id. */
    int n_ovf = 0;
    for (int e = 0; e < E; ++e)
        if (ovf[e] > 0) { order[n_ovf].ovf = (int32_t)ovf[e]; order[n_ovf].e = e; ++n_ovf; }
    qsort(order, (size_t)n_ovf, sizeof(orc_ovf), orc_ovf_cmp);

    /* Greedy: each chunk goes to the eligible rank with most spare capacity,
     * min(remaining, spare) tokens.  The stated rule places the experts one
     * after the other in the fixed order; with ORC_REQUEUE the next chunk is
     * always for the expert with the largest remaining overflow.  Experts
     * still holding overflow when no rank is eligible are "stuck". */
    int n_stuck = 0;
    for (int e = 0; e < E; ++e) rem_e[e] = ovf[e];
    int m_next = 0;                       /* fixed order: next expert to place */
    for (;;) {
        int e = -1;
        if (variant & ORC_REQUEUE) {
            for (int x = 0; x < E; ++x)   /* largest remaining overflow, ties to lower id */
                if (rem_e[x] > 0 && (e < 0 || rem_e[x] > rem_e[e])) e = x;
        } else {
            while (m_next < n_ovf && rem_e[order[m_next].e] == 0) ++m_next;
            if (m_next < n_ovf) e = order[m_next].e;
        }
        if (e < 0) break;                 /* every overflow placed */
        int h = e / H;
        int best = -1;
        for (int r = 0; r < N; ++r) {
            if (used[r] >= R || Q - cur[r] <= 0) continue;   /* not eligible */
            if (best < 0 || Q - cur[r] > Q - cur[best]) best = r;   /* ties keep lowest r */
        }
        if (best < 0) {                   /* slots ran out; none becomes eligible again */
            flags |= 1;
            break;
        }
        if (best == h) { rc = ORC_INVARIANT; goto done; }  /* home is full whenever ovf > 0 */
        for (int a = 0; a < n_asg; ++a)                      /* one replica of e per rank */
            if (asg_e[a] == e && asg_s[a] / HR == best) { rc = ORC_INVARIANT; goto done; }
        int64_t spare = Q - cur[best];
        int64_t c = rem_e[e] < spare ? rem_e[e] : spare;
        asg_e[n_asg] = e;
        asg_s[n_asg] = best * HR + H + used[best];
        asg_c[n_asg] = c;
        ++n_asg;
        used[best] += 1;
        cur[best] += c;
        rem_e[e] -= c;
    }
    /* The stuck experts, in the order the greedy would have visited them:
     * the fixed order, or (requeue) largest remaining first, ties lower id. */
    if (variant & ORC_REQUEUE) {
        for (;;) {
            int e = -1;
            for (int x = 0; x < E; ++x) {
                int taken = 0;
                for (int k = 0; k < n_stuck; ++k) taken |= stuck[k] == x;
                if (!taken && rem_e[x] > 0 && (e < 0 || rem_e[x] > rem_e[e])) e = x;
            }
            if (e < 0) break;
            stuck[n_stuck++] = e;
        }
    } else {
        for (int m = 0; m < n_ovf; ++m)
            if (rem_e[order[m].e] > 0) stuck[n_stuck++] = order[m].e;
    }
    /* Their remainders: on the home slot (the stated rule), or spread token by
     * token over the expert's replicas (home first, then allocation order),
     * each token to the replica whose rank has the lowest load. */
    for (int k = 0; k < n_stuck; ++k) {
        int e = stuck[k], h = e / H;
        if (!(variant & ORC_SPREAD)) {
            home_quota[e] += rem_e[e];
            cur[h] += rem_e[e];
            rem_e[e] = 0;
            continue;
        }
        while (rem_e[e] > 0) {
            int best_a = -1;              /* -1: the home replica */
            int64_t best_load = cur[h];
            for (int a = 0; a < n_asg; ++a) {
                if (asg_e[a] != e) continue;
                int r = asg_s[a] / HR;
                if (cur[r] < best_load) { best_load = cur[r]; best_a = a; }
            }
            if (best_a < 0) { home_quota[e] += 1; cur[h] += 1; }
            else { asg_c[best_a] += 1; cur[asg_s[best_a] / HR] += 1; }
            rem_e[e] -= 1;
        }
    }

    /* Slot table. */
    for (int s = 0; s < S; ++s) { slot_expert[s] = -1; slot_quota[s] = 0; }
    for (int e = 0; e < E; ++e) {
        int s = (e / H) * HR + (e % H);
        slot_expert[s] = e;
        slot_quota[s] = (int32_t)home_quota[e];
    }
    for (int a = 0; a < n_asg; ++a) {
        slot_expert[asg_s[a]] = asg_e[a];
        slot_quota[asg_s[a]] = (int32_t)asg_c[a];
    }

    /* Replica lists: home first, then redundant slots in allocation order;
     * rep_cum is the exclusive prefix of the replicas' quotas. */
    int pos = 0, M = 0;
    for (int e = 0; e < E; ++e) {
        rep_off[e] = pos;
        rep_slot[pos] = (e / H) * HR + (e % H);
        rep_cum[pos] = 0;
        int64_t cum = home_quota[e];
        ++pos;
        int nred = 0;
        for (int a = 0; a < n_asg; ++a) {
            if (asg_e[a] != e) continue;
            rep_slot[pos] = asg_s[a];
            rep_cum[pos] = (int32_t)cum;
            cum += asg_c[a];
            ++pos;
            ++nred;
        }
        if (cum != load[e]) { rc = ORC_INVARIANT; goto done; }   /* conservation */
        if (nred > 0) rep_experts[M++] = e;
    }
    rep_off[E] = pos;
    for (int p = pos; p < E + NR; ++p) { rep_slot[p] = -1; rep_cum[p] = -1; }
    for (int m = M; m < E; ++m) rep_experts[m] = -1;

    int64_t max_before = 0, max_after = 0;
    for (int r = 0; r < N; ++r) {
        int64_t before = 0;
        for (int e = r * H; e < (r + 1) * H; ++e) before += load[e];
        rank_load_before[r] = (int32_t)before;
        rank_load_after[r] = (int32_t)cur[r];
        if (before > max_before) max_before = before;
        if (cur[r] > max_after) max_after = cur[r];
    }
    info[0] = (int32_t)Q;
    info[1] = (int32_t)L;
    info[2] = flags;
    info[3] = M;
    info[4] = n_asg;
    info[5] = (int32_t)max_before;
    info[6] = (int32_t)max_after;
    info[7] = 0;

done:
    free(cur); free(used); free(home_quota); free(ovf); free(order);
    free(asg_e); free(asg_s); free(asg_c); free(rem_e); free(stuck);
    return rc;
}

int ue_oracle_plan(int E, int N, int R, const int32_t *load,
                   int32_t *slot_expert, int32_t *slot_quota,
                   int32_t *rep_off, int32_t *rep_slot, int32_t *rep_cum,
                   int32_t *rep_experts,
                   int32_t *rank_load_before, int32_t *rank_load_after,
                   int32_t *info)
{
    return ue_oracle_plan_ex(E, N, R, load, 0, slot_expert, slot_quota, rep_off, rep_slot, rep_cum,
                             rep_experts, rank_load_before, rank_load_after, info);
}

/* ---- step 3: routing expansion -------------------------------------------
 * The j-th occurrence (0-based, token-major (t, k) order) of expert e goes to
 * the replica i of e with rep_cum[i] <= j < rep_cum[i] + quota of replica i.
 */
int ue_oracle_reroute(const int32_t *ids, int64_t T, int K, int E,
                      const int32_t *rep_off, const int32_t *rep_slot,
                      const int32_t *rep_cum, const int32_t *slot_quota,
                      int32_t *phys)
{
    if (T < 0 || K < 1 || E < 1) return ORC_BAD_ARG;
    int64_t *occ = calloc((size_t)E, sizeof(int64_t));
    if (!occ) return ORC_BAD_ARG;
    int rc = ORC_OK;
    for (int64_t t = 0; t < T; ++t) {
        for (int k = 0; k < K; ++k) {
            int64_t x = t * K + k;
            int32_t e = ids[x];
            if (e < 0 || e >= E) { phys[x] = -1; continue; }
            int64_t j = occ[e]++;
            int found = -1;
            for (int i = rep_off[e]; i < rep_off[e + 1]; ++i) {
                int64_t lo = rep_cum[i], q = slot_quota[rep_slot[i]];
                if (lo <= j && j < lo + q) { found = i; break; }
            }
            if (found < 0) { rc = ORC_INVARIANT; phys[x] = -1; continue; }
            phys[x] = rep_slot[found];
        }
    }
    free(occ);
    return rc;
}

/* ---- after step 3: dispatch layout -----------------------------------------
 * Routing expansion hands its physical routing to token dispatch, which groups
 * the assignments by physical slot before expert compute.  The layout:
 *   slot_off[s]  = number of valid assignments routed to slots below s
 *                  (slot_off[S] = every valid assignment);
 *   src_index    = for s = 0, 1, ..., S-1 in turn, the flat indices x = t*K + k
 *                  with phys[x] = s, in increasing x (a stable counting sort of
 *                  the assignments by slot);
 *   gates_out[p] = gates[src_index[p]] when gates is given.
 * Assignments with phys[x] = -1 (invalid ids) are not dispatched; the entries
 * of src_index / gates_out past slot_off[S] are left untouched.
 */
int ue_oracle_dispatch(const int32_t *phys, int64_t L, int S, const float *gates,
                       int32_t *slot_off, int32_t *src_index, float *gates_out)
{
    if (L < 0 || S < 1) return ORC_BAD_ARG;
    int64_t *cnt = calloc((size_t)S, sizeof(int64_t));
    if (!cnt) return ORC_BAD_ARG;
    for (int64_t x = 0; x < L; ++x) {
        int32_t s = phys[x];
        if (s == -1) continue;
        if (s < 0 || s >= S) { free(cnt); return ORC_BAD_ARG; }
        cnt[s]++;
    }
    int64_t run = 0;
    for (int s = 0; s < S; ++s) {
        slot_off[s] = (int32_t)run;
        int64_t c = cnt[s];
        cnt[s] = run;                    /* from here on: next free position of slot s */
        run += c;
    }
    slot_off[S] = (int32_t)run;
    for (int64_t x = 0; x < L; ++x) {
        int32_t s = phys[x];
        if (s == -1) continue;
        int64_t p = cnt[s]++;
        src_index[p] = (int32_t)x;
        if (gates) gates_out[p] = gates[x];
    }
    free(cnt);
    return ORC_OK;
}

/* ---- step 4: replica weight sync ------------------------------------------
 * Every filled redundant slot s (slot_expert[s] = e >= 0, s % (H+R) >= H)
 * receives a copy of e's home slot.  Slot s starts at byte s * slot_stride of
 * W; the first nbytes bytes of each slot are copied (nbytes = the slot size
 * for a full sync, less for a bounded sample).
 */
int ue_oracle_sync(uint8_t *W, int64_t slot_stride, int64_t nbytes,
                   int E, int N, int R, const int32_t *slot_expert)
{
    if (E < 1 || N < 1 || R < 0 || E % N != 0 || nbytes > slot_stride || nbytes < 0) return ORC_BAD_ARG;
    const int H = E / N, HR = H + R, S = N * HR;
    for (int s = 0; s < S; ++s) {
        int e = slot_expert[s];
        if (s % HR < H || e < 0) continue;
        if (e >= E) return ORC_BAD_ARG;
        int64_t home = (int64_t)(e / H) * HR + (e % H);
        memcpy(W + (int64_t)s * slot_stride, W + home * slot_stride, (size_t)nbytes);
    }
    return ORC_OK;
}

/* ---- step 4, incremental form ---------------------------------------------
 * Within one training step the expert weights do not change between
 * microbatches, so a redundant slot that held expert e under the previous
 * microbatch's plan (prev_slot_expert[s] = e) already holds e's home weights:
 * only filled redundant slots whose expert differs from prev are copied.  With
 * prev_slot_expert NULL every filled redundant slot is copied (a full sync,
 * as after the optimizer step).  *copied = number of slots copied.
 */
int ue_oracle_sync_delta(uint8_t *W, int64_t slot_stride, int64_t nbytes,
                         int E, int N, int R, const int32_t *slot_expert,
                         const int32_t *prev_slot_expert, int64_t *copied)
{
    if (E < 1 || N < 1 || R < 0 || E % N != 0 || nbytes > slot_stride || nbytes < 0) return ORC_BAD_ARG;
    const int H = E / N, HR = H + R, S = N * HR;
    int64_t n = 0;
    for (int s = 0; s < S; ++s) {
        int e = slot_expert[s];
        if (s % HR < H || e < 0) continue;
        if (e >= E) return ORC_BAD_ARG;
        if (prev_slot_expert && prev_slot_expert[s] == e) continue;
        int64_t home = (int64_t)(e / H) * HR + (e % H);
        memcpy(W + (int64_t)s * slot_stride, W + home * slot_stride, (size_t)nbytes);
        ++n;
    }
    if (copied) *copied = n;
    return ORC_OK;
}

/* ---- weight restore in backward ----------------------------------------------
 * "How dots-infra/ultraep works" (summary paragraph): after planning, weight
 * sync and routing expansion before expert execution, UltraEP restores
 * weights and reduces replica gradients during backward.  Reading taken here:
 * the layers (and microbatches) share the redundant slots, so when backward
 * reaches a layer its redundant slots hold the replicas of another plan, the
 * one last synced into them (held_slot_expert), and the expert backward of the
 * layer needs the layer's own forward replicas back.  So every redundant slot
 * that the layer's plan fills with expert e (target_slot_expert[s] = e >= 0)
 * and that does not hold e already receives e's home slot; slots the target
 * leaves empty, and home slots, are untouched.  held_slot_expert NULL: what
 * the slots hold is unknown, and every filled redundant slot of the target is
 * copied.  *copied = the number of slots copied.
 */
int ue_oracle_sync_restore(uint8_t *W, int64_t slot_stride, int64_t nbytes, int E, int N, int R,
                           const int32_t *target_slot_expert, const int32_t *held_slot_expert,
                           int64_t *copied)
{
    if (E < 1 || N < 1 || R < 0 || E % N != 0 || nbytes > slot_stride || nbytes < 0) return ORC_BAD_ARG;
    const int H = E / N, HR = H + R;
    int64_t n = 0;
    for (int r = 0; r < N; ++r)
        for (int u = 0; u < R; ++u) {
            const int s = r * HR + H + u;                 /* rank r's u-th redundant slot */
            const int e = target_slot_expert[s];
            if (e < 0) continue;                           /* empty under the target: left as it is */
            if (e >= E) return ORC_BAD_ARG;
            if (held_slot_expert && held_slot_expert[s] == e) continue;   /* holds e already */
            const int64_t home_slot = (int64_t)(e / H) * HR + e % H;
            memcpy(W + (int64_t)s * slot_stride, W + home_slot * slot_stride, (size_t)nbytes);
            ++n;
        }
    if (copied) *copied = n;
    return ORC_OK;
}

/* ---- step 4 across GPUs: relay against fan-out overload -------------------
 * The news summary ("Comment fonctionne l'équilibrage en 300 microsecondes")
 * streams expert states between GPUs with a relay mechanism against fan-out
 * overload.  Reading taken here: the N ranks are spread over G GPUs, GPU g
 * holding ranks [g*N/G, (g+1)*N/G) and so slots [g*SG, (g+1)*SG), SG = S/G.
 * For an expert e, its consumers c_0 < c_1 < ... < c_{f-1} are the GPUs other
 * than its home GPU that hold a filled redundant slot of e.  The expert's
 * bytes are cut into f parts of q = 16 * ceil(nbytes / (16 f)) bytes, part j
 * = [j q, min((j+1) q, nbytes)) (trailing parts may be empty).
 *   round 0: consumer c_j receives part j from the home slot; the home GPU
 *            fills its own redundant slots of e from the home slot;
 *   round 1: consumer c_i receives every part j != i from consumer c_j
 *            (c_j's lowest slot holding e, filled in round 0).
 * A received range is written into every redundant slot of e on the GPU.  So
 * the home sends each byte once whatever f is (a scatter, then an all-gather
 * among the consumers).  Rounds: 1 when G <= 2 (f <= 1), else 2.
 * round = -1 is the direct form: every redundant slot of e is filled from the
 * home slot (the single-GPU sync), the home sending nbytes to each consumer.
 * Only destinations on GPU dst_gpu are written (every GPU when dst_gpu = -1).
 * egress[G] (optional) receives the bytes each GPU sent to other GPUs in this
 * round (for the destinations written).
 */
int ue_oracle_relay_rounds(int G)
{
    return G <= 2 ? 1 : 2;
}

int ue_oracle_sync_relay(uint8_t *W, int64_t slot_stride, int64_t nbytes,
                         int E, int N, int R, const int32_t *slot_expert,
                         int G, int round, int dst_gpu, int64_t *egress)
{
    if (E < 1 || N < 1 || R < 0 || E % N != 0 || nbytes > slot_stride || nbytes < 0) return ORC_BAD_ARG;
    if (G < 1 || N % G != 0 || round < -1 || round > 1 || dst_gpu < -1 || dst_gpu >= G) return ORC_BAD_ARG;
    const int H = E / N, HR = H + R, S = N * HR, SG = S / G;
    int *cons = (int *)malloc(sizeof(int) * (size_t)G);
    int *first = (int *)malloc(sizeof(int) * (size_t)G);
    if (!cons || !first) { free(cons); free(first); return ORC_BAD_ARG; }
    if (egress) memset(egress, 0, sizeof(int64_t) * (size_t)G);
    for (int s = 0; s < S; ++s)
        if (slot_expert[s] >= E) { free(cons); free(first); return ORC_BAD_ARG; }
    for (int e = 0; e < E; ++e) {
        const int home = (e / H) * HR + (e % H);
        const int hg = home / SG;
        /* consumers in increasing GPU id, with each one's lowest slot of e */
        int f = 0;
        for (int g = 0; g < G; ++g) {
            int lo = -1;
            for (int s = g * SG; s < (g + 1) * SG && lo < 0; ++s)
                if (s % HR >= H && slot_expert[s] == e) lo = s;
            if (lo >= 0 && g != hg) { cons[f] = g; first[f] = lo; ++f; }
        }
        const int64_t q = f > 0 ? 16 * ((nbytes + 16 * (int64_t)f - 1) / (16 * (int64_t)f)) : 0;
        /* every GPU holding e receives, in this round, a list of (source slot, byte range) */
        for (int g = 0; g < G; ++g) {
            if (dst_gpu >= 0 && g != dst_gpu) continue;
            int i = -1;                                  /* g's consumer index */
            for (int j = 0; j < f; ++j) if (cons[j] == g) i = j;
            if (g != hg && i < 0) continue;
            for (int j = 0; j < (g == hg ? 1 : f); ++j) {
                int src;
                int64_t lo, hi;
                if (g == hg) {                           /* home GPU: its own replicas */
                    if (round > 0) break;
                    src = home; lo = 0; hi = nbytes;
                } else if (round < 0) {                  /* direct: the whole slot, once */
                    if (j > 0) break;
                    src = home; lo = 0; hi = nbytes;
                } else if (round == 0) {                 /* scatter: its own part from home */
                    if (j != i) continue;
                    src = home; lo = j * q; hi = (j + 1) * q;
                } else {                                 /* all-gather: the other parts */
                    if (j == i) continue;
                    src = first[j]; lo = j * q; hi = (j + 1) * q;
                }
                if (hi > nbytes) hi = nbytes;
                if (lo >= hi) continue;
                int wrote = 0;
                for (int s = g * SG; s < (g + 1) * SG; ++s) {
                    if (s % HR < H || slot_expert[s] != e) continue;
                    memcpy(W + (int64_t)s * slot_stride + lo, W + (int64_t)src * slot_stride + lo, (size_t)(hi - lo));
                    wrote = 1;
                }
                const int sg = src / SG;
                if (wrote && sg != g && egress) egress[sg] += hi - lo;
            }
        }
    }
    free(cons);
    free(first);
    return ORC_OK;
}

/* ---- step 5: replica gradient reduction -----------------------------------
 * For each expert e with redundant replicas, in replica order i = 1, 2, ...:
 *     master[e][x] = master[e][x] + float(grad[g(i)][x])
 * where g(i) is the replica-gradient row of redundant slot rep_slot[i]:
 * slot r*(H+R) + H + u  ->  row r*R + u.  master rows have stride `mstride`
 * floats, gradient rows `gstride` elements; n elements of each are reduced.
 */
static float orc_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

int ue_oracle_grad_reduce(float *master, int64_t mstride, const void *grads,
                          int grad_is_bf16, int64_t gstride, int64_t n,
                          int E, int N, int R,
                          const int32_t *rep_off, const int32_t *rep_slot)
{
    if (E < 1 || N < 1 || R < 0 || E % N != 0 || n < 0) return ORC_BAD_ARG;
    const int H = E / N, HR = H + R;
    for (int e = 0; e < E; ++e) {
        float *m = master + (int64_t)e * mstride;
        for (int i = rep_off[e] + 1; i < rep_off[e + 1]; ++i) {
            int s = rep_slot[i];
            int r = s / HR, u = s % HR - H;
            if (u < 0 || u >= R) return ORC_INVARIANT;
            int64_t row = (int64_t)r * R + u;
            if (grad_is_bf16) {
                const uint16_t *g = (const uint16_t *)grads + row * gstride;
                for (int64_t x = 0; x < n; ++x) m[x] = m[x] + orc_bf16_to_f32(g[x]);
            } else {
                const float *g = (const float *)grads + row * gstride;
                for (int64_t x = 0; x < n; ++x) m[x] = m[x] + g[x];
            }
        }
    }
    return ORC_OK;
}
