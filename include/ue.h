/*
 * ue.h - C ABI of libue.so, a B200 (sm_100a) implementation of the per-layer,
 * per-microbatch hot path of UltraEP's real-time MoE expert balancer
 * (arXiv 2606.04101, "UltraEP: Unleash MoE Training and Inference on
 * Rack-Scale Nodes with Near-Optimal Load Balancing").
 *
 * The pipeline runs right after gating (UltraEP news summary, "Comment
 * fonctionne l'équilibrage en 300 microsecondes"): load computation ->
 * placement planning -> routing expansion -> replica weight sync, and, in the
 * backward pass, replica gradient reduction ("How dots-infra/ultraep works",
 * component list "GPU operations" and its "Connections").  All N
 * expert-parallel (EP) ranks are simulated as partitions of one GPU's memory.
 *
 * Layout shared by every call (E experts, N ranks, H = E / N, R redundant
 * slots per rank, S = N * (H + R) physical slots):
 *   - expert e is homed on rank e / H in local slot e % H;
 *   - physical slot id = r * (H + R) + s; local slots s in [H, H + R) are the
 *     rank's redundant (replica) slots;
 *   - token t belongs to source rank t / (T / N); ids are token-major [T][K].
 *
 * Conventions.
 *   - Every array is caller-owned device memory unless stated; the library
 *     allocates nothing per call.  `stream` is a cudaStream_t (NULL = legacy
 *     default stream).  Calls are asynchronous and never synchronize the host.
 *   - Host-detectable errors (null or misaligned pointers, sizes out of
 *     range) return UE_ERR_INVALID_ARG before any launch; outputs are then
 *     left untouched.  ue_last_error() gives a one-line reason.
 *   - Device-detected bad input (an id outside [0, E)) never traps: the id is
 *     not counted, its rerouted slot is -1, and ue_load reports it per rank.
 *   - Limits: 1 <= E <= 1024, 1 <= N <= 1024, E % N == 0, 0 <= R,
 *     N * R <= 4096, 1 <= K, T % N == 0, T * K <= 2^30.
 */
#ifndef UE_H
#define UE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    UE_OK = 0,
    UE_ERR_INVALID_ARG = 1,   /* rejected before launch; outputs untouched */
    UE_ERR_CUDA = 2,          /* a CUDA runtime call or launch failed */
    UE_ERR_UNSUPPORTED = 3,   /* device is not sm_100 or lacks a needed feature */
    UE_ERR_DEVICE = 4         /* a kernel gave up a bounded wait (see ue_ctx_device_error) */
} ue_status;

/* Opaque per-device context: caches device properties and kernel attributes
 * and owns a device status word for bounded-wait failures and a 16 MiB device
 * workspace, both allocated by ue_ctx_create.  The workspace holds the
 * per-piece histograms that ue_rebalance(_ex) and ue_reroute(_shard) pass
 * from their load pass to their reroute pass when a CTA's share of a rank's
 * ids exceeds what the reroute keeps on chip (many ranks or many tokens per
 * rank), and the expert loads that the load pass of ue_rebalance,
 * ue_rebalance_ex and ue_rebalance_dispatch sums for their planner (zeros
 * between calls: the planner writes them back); such calls on one context
 * must not overlap on the GPU (issue them on one stream, or order the
 * streams).  Capturing them in a CUDA graph and replaying it is fine. */
typedef struct ue_ctx ue_ctx;

/* Problem shape.  H = E / N and S = N * (H + R) are derived. */
typedef struct {
    int32_t E;   /* experts */
    int32_t N;   /* simulated EP ranks */
    int32_t R;   /* redundant (replica) slots per rank */
    int32_t K;   /* top-k experts per token */
    int64_t T;   /* tokens in the microbatch (all ranks) */
} ue_config;

/* The placement plan: device arrays, caller-allocated with the sizes below
 * (ue_plan_sizes), written by ue_plan and read by ue_reroute, ue_sync and
 * ue_grad_reduce.  "Placement planning -> Native Manager: placement plan"
 * ("How dots-infra/ultraep works", Connections). */
typedef struct {
    int32_t *slot_expert;       /* [S]    expert held by each physical slot, -1 = empty       */
    int32_t *slot_quota;        /* [S]    tokens routed to each slot                          */
    int32_t *rep_off;           /* [E+1]  replicas of e are entries rep_off[e] .. rep_off[e+1]-1 */
    int32_t *rep_slot;          /* [E+N*R] slot of each replica: home first, then allocation order; -1 tail */
    int32_t *rep_cum;           /* [E+N*R] exclusive prefix of the replicas' quotas; -1 tail   */
    int32_t *rep_experts;       /* [E]    experts with >= 1 redundant replica, increasing id; -1 tail */
    int32_t *load;              /* [E]    exact load: occurrences of e in the microbatch      */
    int32_t *rank_off;          /* [N*E]  occurrences of e in the tokens of ranks < r          */
    int32_t *rank_load_before;  /* [N]    tokens routed to rank r's home experts              */
    int32_t *rank_load_after;   /* [N]    tokens rank r serves under the plan                 */
    int32_t *info;              /* [8]    Q, L, flags (bit 0: slots ran out), M = #rep_experts,
                                          filled redundant slots, max before, max after, 0    */
} ue_plan_buffers;

/* Element counts (int32 entries) of the 11 ue_plan_buffers arrays, in field
 * order, for a configuration.  Host only. */
ue_status ue_plan_sizes(const ue_config *cfg, int64_t sizes[11]);

/* Create a context on CUDA device `device` (made current for the call). */
ue_status ue_ctx_create(int device, ue_ctx **out);
ue_status ue_ctx_destroy(ue_ctx *ctx);

/* Copy the context's device status word to *host_word (synchronizes
 * `stream`) and clear it.  Bit 0: a kernel gave up a bounded wait; bit 1:
 * ue_dispatch met ids that do not match the plan. */
ue_status ue_ctx_device_error(ue_ctx *ctx, int32_t *host_word, void *stream);

/* Bound of every wait inside the kernels that stream through rings of bulk
 * copies - weight sync (ue_sync, ue_sync_delta, ue_sync_restore,
 * ue_sync_shard) and gradient reduction (ue_grad_reduce): a copy that has not
 * landed (or a ring slot not released) limit_ns nanoseconds (GPU global timer)
 * after the kernel began to wait for it makes the kernel give up - it sets bit
 * 0 of the status word, waits for its other copies in flight (each wait again
 * bounded by limit_ns) and returns; that call's outputs are then incomplete,
 * and a copy that never lands leaves the device state undefined.  Default
 * 2 s; limit_ns in [1000, 6e10].  Host only; affects later calls.
 *   flags  UE_WAIT_STALL_ONCE (diagnostic, for testing the way out): the next
 *          such call on this context makes one party of its first CTA wait
 *          once on a barrier that nothing completes (after the first copies
 *          are in flight), so that this wait runs out; the flag then clears. */
#define UE_WAIT_STALL_ONCE 1
ue_status ue_ctx_set_wait_limit(ue_ctx *ctx, int64_t limit_ns, int32_t flags);

/* ---- step 1: load computation ----------------------------------------------
 * "Load computation" (csrc/kernels/load_compute.cu in the component list of
 * "How dots-infra/ultraep works"; "exact-load" in the arXiv abstract).
 *   ids    [T][K] int32, 16-byte aligned: post-gating top-k expert ids.
 *   counts [N][E] int32 out: counts[r][e] = #{(t,k): t in rank r, ids[t][k] = e}.
 *   bad    [N] int32 out, may be NULL: ids of rank r's tokens outside [0, E).
 * Every entry of counts (and bad) is overwritten; no pre-zeroing needed. */
ue_status ue_load(ue_ctx *ctx, const ue_config *cfg, const int32_t *ids,
                  int32_t *counts, int32_t *bad, void *stream);

/* ---- step 2: quota-driven placement planning ---------------------------------
 * "Placement planning" (csrc/kernels/placement.cu); the quota-driven scheduler
 * of the news summary.  From counts [N][E] (as written by ue_load):
 *   load[e] = sum_r counts[r][e], L = sum_e load[e], Q = ceil(L / N);
 *   home pass in increasing e: the home rank takes min(load, Q - current);
 *   overflow experts, largest overflow first (ties: lower id), are placed
 *   chunk by chunk on the rank with most spare capacity Q - current (ties:
 *   lowest rank) among ranks with a free redundant slot and spare > 0, each
 *   chunk min(remaining, spare); at most R replicas per rank; if no rank is
 *   eligible the remainder stays on the home slot (flag bit 0).
 * Writes every array of *plan (the buffers themselves are read from host
 * memory; their contents are device memory). */
ue_status ue_plan(ue_ctx *ctx, const ue_config *cfg, const int32_t *counts,
                  const ue_plan_buffers *plan, void *stream);

/* Plan variants for the two points the rule leaves open (bit flags for
 * ue_plan_ex / ue_rebalance_ex; 0 = ue_plan):
 *   UE_PLAN_REQUEUE  the overflow is a priority queue: after every chunk the
 *                    expert with the largest remaining overflow (ties: lower
 *                    id) is placed next, instead of each expert being placed
 *                    fully in the order fixed after the home pass;
 *   UE_PLAN_SPREAD   when slots run out, each stuck expert's remainder (in
 *                    visit order) goes token by token to the replica whose rank
 *                    has the lowest load (ties: earlier replica, home first)
 *                    instead of staying on the home slot.
 * Everything else (quota, home pass, eligibility, chunk size, replica order,
 * cumulative quotas, outputs) is as in ue_plan. */
#define UE_PLAN_REQUEUE 1
#define UE_PLAN_SPREAD 2
ue_status ue_plan_ex(ue_ctx *ctx, const ue_config *cfg, const int32_t *counts,
                     const ue_plan_buffers *plan, int variant, void *stream);

/* ---- step 3: routing expansion ---------------------------------------------
 * "Routing expansion" (csrc/kernels/reroute.cu; "Routing expansion -> Token
 * dispatch: physical routing").  The j-th occurrence (0-based, token-major
 * (t, k) order) of expert e goes to replica i of e with
 * rep_cum[i] <= j < rep_cum[i] + quota(i):  phys[t][k] = rep_slot[i].
 *   ids  [T][K] int32, 16-byte aligned (the ids the plan was computed from).
 *   phys [T][K] int32 out; -1 for ids outside [0, E). */
ue_status ue_reroute(ue_ctx *ctx, const ue_config *cfg, const int32_t *ids,
                     const ue_plan_buffers *plan, int32_t *phys, void *stream);

/* Routing expansion without a context, for callers that cannot allocate
 * device memory - an engine that reserves its whole device-memory budget in
 * its own pool at start-up, or a caller in a region of its framework where
 * allocation is not allowed - and so cannot create a ue_ctx (ue_ctx_create
 * allocates).  The pages have no counterpart: it is an interface of this
 * library.  Same arguments and the same phys as ue_reroute, on the current
 * device; it always takes the reroute over pieces, with its scratch (piece
 * counters and per-piece occurrence rows) in a 4 MiB device array that the
 * library holds on every GPU that loads it until the process exits.  It calls
 * no allocating routine.
 *   - Limit: 2 * N * (E + 1) + 64 <= 2^20 ints (else UE_ERR_INVALID_ARG,
 *     phys untouched), plus the limits above.
 *   - The first call on a device sets that device up (looks up the array's
 *     device address, sets the kernels' shared-memory limits); make that first
 *     call before any stream capture.
 *   - Every call shares the array and leaves its contents behind (each call
 *     clears the counters it needs at 0 and overwrites the rows it reads):
 *     calls that overlap on the GPU race - issue them on one stream, or order
 *     the streams. */
ue_status ue_reroute_static(const ue_config *cfg, const int32_t *ids, const ue_plan_buffers *plan,
                            int32_t *phys, void *stream);

/* Steps 1-3 back to back on one stream (three launches). */
ue_status ue_rebalance(ue_ctx *ctx, const ue_config *cfg, const int32_t *ids,
                       int32_t *counts, int32_t *bad, const ue_plan_buffers *plan,
                       int32_t *phys, void *stream);

/* ue_rebalance with a plan variant (UE_PLAN_REQUEUE | UE_PLAN_SPREAD bits). */
ue_status ue_rebalance_ex(ue_ctx *ctx, const ue_config *cfg, const int32_t *ids,
                          int32_t *counts, int32_t *bad, const ue_plan_buffers *plan,
                          int32_t *phys, int variant, void *stream);

/* ---- dispatch layout (after step 3) ------------------------------------------
 * Routing expansion hands the physical routing to token dispatch, which groups
 * the assignments by physical slot for expert compute ("Routing expansion ->
 * Token dispatch: physical routing", "Token dispatch -> Expert compute:
 * dispatches tokens" in "How dots-infra/ultraep works").  Layout:
 *   slot_off[s]  = assignments routed to slots below s (exclusive prefix of
 *                  plan.slot_quota; slot_off[S] = all valid assignments);
 *   src_index[p] for p in [slot_off[s], slot_off[s+1]): the flat indices
 *                  x = t*K + k with phys[x] = s, increasing (stable grouping);
 *   gates_out[p] = gates[src_index[p]] (bit copy) when gates is given.
 * Ids outside [0, E) are not dispatched; entries past slot_off[S] are left
 * untouched. */
typedef struct {
    const float *gates;   /* [T*K] fp32 gate of each (t, k), or NULL                    */
    int32_t *slot_off;    /* [S+1] out                                                  */
    int32_t *src_index;   /* [T*K] out                                                  */
    float *gates_out;     /* [T*K] out; required when gates is given, else ignored      */
} ue_dispatch_buffers;

/* Routing expansion with the dispatch layout: writes phys exactly as
 * ue_reroute does, plus *disp.  ids must be the ids the plan was computed
 * from: an assignment that falls outside its slot's segment (a plan from other
 * ids) is not written and sets bit 1 (value 2) of the context's device status
 * word (ue_ctx_device_error). */
ue_status ue_dispatch(ue_ctx *ctx, const ue_config *cfg, const int32_t *ids,
                      const ue_plan_buffers *plan, int32_t *phys,
                      const ue_dispatch_buffers *disp, void *stream);

/* Steps 1-3 with the dispatch layout, back to back on one stream (three launches). */
ue_status ue_rebalance_dispatch(ue_ctx *ctx, const ue_config *cfg, const int32_t *ids,
                                int32_t *counts, int32_t *bad, const ue_plan_buffers *plan,
                                int32_t *phys, const ue_dispatch_buffers *disp, void *stream);

/* ---- step 4: replica weight sync ---------------------------------------------
 * "Replica weight sync" (csrc/kernels/weight_sync.cu; "persistent tile
 * streaming" with a relay against fan-out overload in the news summary).
 * For every filled redundant slot s holding expert e, slot s receives a byte
 * copy of e's home slot.  Each home tile is read once and written to all of
 * that expert's replicas.
 *   weights     device base of S slots, slot s at byte s * slot_bytes,
 *               16-byte aligned; home slots are read, filled redundant slots
 *               written, empty slots untouched.
 *   slot_bytes  bytes per slot (3 bf16 matrices: 6 * rows * cols), multiple of 16. */
ue_status ue_sync(ue_ctx *ctx, const ue_config *cfg, void *weights, int64_t slot_bytes,
                  const ue_plan_buffers *plan, void *stream);

/* Incremental weight sync for the microbatches of one training step, whose
 * expert weights do not change between microbatches: a filled redundant slot
 * whose expert equals prev_slot_expert[s] (the previous microbatch's
 * plan.slot_expert, [S] device memory, read only) already holds that expert's
 * weights and is not written; every other filled redundant slot is copied as
 * in ue_sync.  prev_slot_expert = NULL gives the full sync (the first
 * microbatch after an optimizer step). */
ue_status ue_sync_delta(ue_ctx *ctx, const ue_config *cfg, void *weights, int64_t slot_bytes,
                        const ue_plan_buffers *plan, const int32_t *prev_slot_expert, void *stream);

/* Weight restore in backward ("How dots-infra/ultraep works", summary
 * paragraph: UltraEP restores weights and reduces replica gradients during
 * backward).  The layers (and microbatches) share the redundant slots, so when
 * backward reaches a layer its slots hold the replicas of another plan; this
 * call brings back the layer's forward replicas before its expert backward:
 * every filled redundant slot of `plan` (the layer's saved forward plan) whose
 * expert differs from held_slot_expert[s] receives a byte copy of its expert's
 * home slot; other slots are untouched.
 *   held_slot_expert  [S] device memory, read only: the expert each slot holds
 *                     now (the slot_expert of the plan last synced into it, or
 *                     built by the caller slot by slot); NULL = unknown, every
 *                     filled redundant slot of plan is copied.
 * The same operation as ue_sync_delta with the saved plan as its target; the
 * weights, slot_bytes and alignment rules are those of ue_sync. */
ue_status ue_sync_restore(ue_ctx *ctx, const ue_config *cfg, void *weights, int64_t slot_bytes,
                          const ue_plan_buffers *plan, const int32_t *held_slot_expert, void *stream);

/* ---- step 5: replica gradient reduction ------------------------------------
 * "Replica gradient reduction" (csrc/kernels/grad_reduce.cu; "Expert compute
 * -> Replica gradient reduction: replica gradients", "-> MoE framework:
 * master gradients").  For every expert e with redundant replicas, in replica
 * order: master[e][x] = master[e][x] + float(grad[row(i)][x]) (one fp32
 * round-to-nearest add per replica; bf16 widened exactly), where the replica
 * gradient row of redundant slot r*(H+R) + H + u is r*R + u.
 *   master     [E][P] fp32 in/out, 16-byte aligned (rows of unreplicated experts untouched).
 *   grads      [N*R][P] fp32 (grad_dtype 0) or bf16 (grad_dtype 1), 16-byte aligned.
 *   P          elements per expert, multiple of 8. */
ue_status ue_grad_reduce(ue_ctx *ctx, const ue_config *cfg, float *master,
                         const void *grads, int grad_dtype, int64_t P,
                         const ue_plan_buffers *plan, void *stream);

/* ---- across the GPUs of one NVLink domain ----------------------------------
 * The N ranks spread over G GPUs: GPU g holds ranks [g*N/G, (g+1)*N/G), their
 * tokens [g*T/G, (g+1)*T/G) (ids_local [T/G][K]), slots [g*SG, (g+1)*SG) with
 * SG = S / G, the experts [g*E/G, (g+1)*E/G) homed on them (master_local
 * [E/G][P]) and the replica-gradient rows [g*(N/G)*R, (g+1)*(N/G)*R)
 * (N/G*R rows of P elements).  Per microbatch, on every GPU:
 *   ue_load_shard -> all-gather of the counts rows (the caller's collective,
 *   e.g. NCCL) -> ue_plan on the full counts (every GPU computes the same
 *   plan) -> ue_reroute_shard -> ue_sync_shard for each relay round, with a
 *   barrier across GPUs before each round after the first and after the last.
 * In backward, after a barrier (every replica gradient written):
 *   ue_grad_reduce_shard, then a barrier before replica gradients are reused.
 * Peer tables are host arrays of G device pointers, entry h = GPU h's buffer
 * as mapped on the calling GPU (peer access, CUDA IPC or symmetric memory),
 * entry g = the calling GPU's own; each 16-byte aligned.  No kernel waits on
 * another GPU; a copy never uses cluster multicast.  Limits: 1 <= G <= 128,
 * N % G == 0, plus the limits above. */
typedef struct {
    int32_t G;   /* GPUs */
    int32_t g;   /* the calling GPU, 0 <= g < G */
} ue_shard;

/* Step 1 for GPU g's ranks: writes rows [g*N/G, (g+1)*N/G) of counts [N][E]
 * and the same entries of bad [N] (may be NULL); other rows are untouched. */
ue_status ue_load_shard(ue_ctx *ctx, const ue_config *cfg, const ue_shard *shard,
                        const int32_t *ids_local, int32_t *counts, int32_t *bad, void *stream);

/* Step 3 for GPU g's tokens with the plan of the full counts (its rank_off
 * rows for GPU g's ranks are read): phys_local [T/G][K] as ue_reroute's rows
 * [g*T/G, (g+1)*T/G). */
ue_status ue_reroute_shard(ue_ctx *ctx, const ue_config *cfg, const ue_shard *shard,
                           const int32_t *ids_local, const ue_plan_buffers *plan,
                           int32_t *phys_local, void *stream);

/* Relay rounds for G GPUs: 1 when G <= 2, else 2; -1 if G is out of range. */
int32_t ue_relay_rounds(int32_t G);

/* Step 4 across GPUs with the relay against fan-out overload (news summary,
 * "Comment fonctionne l'équilibrage en 300 microsecondes"), as a scatter then
 * an all-gather.  The consumers of expert e are the GPUs other than its home
 * GPU with a filled redundant slot of e, c_0 < c_1 < ... < c_{f-1}; the slot is
 * cut into f parts of q = 16 * ceil(slot_bytes / (16 f)) bytes, part j =
 * [j q, min((j+1) q, slot_bytes)).  Round 0: c_j copies part j from the home
 * slot, and the home GPU fills its own redundant slots of e; round 1: c_i
 * copies every other part j from c_j's lowest slot of e.  A received range is
 * written into every redundant slot of e on the receiving GPU, so the home
 * sends each byte once.  round = -1: the direct form, every consumer copies
 * the whole slot from the home slot (one call instead of the rounds).  This
 * call writes only GPU g's slots (slot_bases[g]) and reads home slots and, in
 * round 1, parts other GPUs received in round 0.  After all rounds every
 * GPU's slots hold what ue_sync gives.
 *   slot_bases  [G] host array of device pointers, each GPU's SG slots of
 *               slot_bytes bytes (multiple of 16). */
ue_status ue_sync_shard(ue_ctx *ctx, const ue_config *cfg, const ue_shard *shard,
                        void *const *slot_bases, int64_t slot_bytes,
                        const ue_plan_buffers *plan, int32_t round, void *stream);

/* Step 5 across GPUs: for every expert e homed on GPU g with redundant
 * replicas, in replica order, master_local[e - g*E/G][x] += float(gradient of
 * the replica), the replica's row read from the GPU holding its slot: row
 * r*R + u of redundant slot r*(H+R) + H + u lives on GPU h = r / (N/G) at local
 * row (r - h*N/G)*R + u of grad_bases[h].  The same adds in the same order as
 * ue_grad_reduce, so the result is bit-identical.
 *   grad_bases  [G] host array of device pointers (may be NULL when R = 0). */
ue_status ue_grad_reduce_shard(ue_ctx *ctx, const ue_config *cfg, const ue_shard *shard,
                               float *master_local, const void *const *grad_bases, int grad_dtype,
                               int64_t P, const ue_plan_buffers *plan, void *stream);

/* Status name, and the reason for the last non-OK status on this thread. */
const char *ue_status_string(ue_status s);
const char *ue_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* UE_H */
