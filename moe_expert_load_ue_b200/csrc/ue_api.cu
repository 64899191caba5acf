// C ABI of libue.so: argument validation, per-device context and launches.
// See include/ue.h for the contract of every entry point.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <new>

#include "ue_internal.cuh"

namespace ue {
cudaError_t set_load_attributes(size_t max_smem);
cudaError_t set_reroute_attributes(size_t max_smem);
cudaError_t set_plan_attributes(size_t max_smem);
cudaError_t set_sync_attributes(size_t max_smem);
cudaError_t set_shard_attributes(size_t max_smem);
cudaError_t set_reroute_pieces_attributes(size_t max_smem);
cudaError_t set_grad_bulk_attributes(size_t max_smem);
}  // namespace ue

struct ue_ctx {
    int device;
    int sms;
    int max_smem;          // opt-in dynamic shared memory per block
    int32_t *dev_err;      // device status word for bounded waits
    int32_t *ws;           // workspace: piece histogram rows of the persistent reroute
    int rp_blocks;         // resident persistent-reroute CTAs per SM as registers allow
    int smem_per_sm;       // shared memory of an SM, and the part each resident CTA reserves
    int smem_reserved;
    int64_t wait_ns;       // bound of one wait in the weight-sync kernels
    int stall_once;        // diagnostic: the next weight sync stalls once (UE_WAIT_STALL_ONCE)
    bool lv_dirty;         // a load grid may have added into the load vector without its planner
};

namespace {
// Workspace of a context (16 MiB): 64 ints of counters (the persistent
// reroute's piece counters, kept at 0 between launches), the expert load
// vector of a fused rebalance (kMaxE ints, zeros between calls: the load grid
// adds into it, its planner reads it and writes the zeros back), then the
// piece rows [N][B + 1][E + 1] of one call from kWsHead on.
constexpr int64_t kWsInts = (int64_t)1 << 22;
constexpr int64_t kWsLoadVec = 64;
constexpr int64_t kWsHead = kWsLoadVec + ue::kMaxE;
// Pieces of the persistent reroute are whole sub-chunks of its CTA (8192 ids:
// 16 per thread), so every warp has work; its per-piece table costs about as
// much as streaming a few thousand ids.
constexpr int64_t kPieceQuantum = 8192;
// Pieces per resident CTA aimed at (they are claimed dynamically; more,
// smaller pieces shorten the tail).
constexpr int kPiecesPerCta = 16;
// Largest CTA share of a rank's ids routed by the rank-per-cluster kernel.
// Measured on B200 over the sweep's shapes: up to 64 Ki ids per share it is
// faster (its first pass overlaps the planner; the persistent kernel pays a
// few microseconds more of fixed cost); from 128 Ki ids the persistent kernel
// is faster, by up to 2x when the quota boundaries crowd into one rank.
constexpr int64_t kClusterShareMax = 65536;
}  // namespace

namespace {

thread_local char g_last_error[512] = "";

ue_status fail(ue_status s, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return s;
}

ue_status cuda_fail(cudaError_t e, const char *what)
{
    return fail(UE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Validates the shape; fills `sh`.  `need_tokens` adds the T/K checks.
ue_status make_shape(const ue_config *cfg, bool need_tokens, ue::Shape *sh)
{
    if (!cfg) return fail(UE_ERR_INVALID_ARG, "config is NULL");
    const ue_config c = *cfg;
    if (c.E < 1 || c.E > ue::kMaxE) return fail(UE_ERR_INVALID_ARG, "E=%d outside [1, %d]", c.E, ue::kMaxE);
    if (c.N < 1 || c.N > ue::kMaxN) return fail(UE_ERR_INVALID_ARG, "N=%d outside [1, %d]", c.N, ue::kMaxN);
    if (c.E % c.N != 0) return fail(UE_ERR_INVALID_ARG, "E=%d is not a multiple of N=%d", c.E, c.N);
    if (c.R < 0 || (int64_t)c.N * c.R > ue::kMaxNR)
        return fail(UE_ERR_INVALID_ARG, "R=%d invalid (need 0 <= R and N*R <= %d)", c.R, ue::kMaxNR);
    if (need_tokens) {
        if (c.K < 1) return fail(UE_ERR_INVALID_ARG, "K=%d < 1", c.K);
        if (c.T < 0 || c.T % c.N != 0)
            return fail(UE_ERR_INVALID_ARG, "T=%lld must be >= 0 and a multiple of N=%d", (long long)c.T, c.N);
        if (c.T * (int64_t)c.K > ((int64_t)1 << 30))
            return fail(UE_ERR_INVALID_ARG, "T*K=%lld exceeds 2^30", (long long)(c.T * c.K));
    }
    sh->E = c.E;
    sh->N = c.N;
    sh->R = c.R;
    sh->K = c.K;
    sh->H = c.E / c.N;
    sh->HR = sh->H + c.R;
    sh->S = c.N * sh->HR;
    sh->NR = c.N * c.R;
    sh->T = c.T;
    sh->per_rank = need_tokens ? (c.T / c.N) * c.K : 0;
    return UE_OK;
}

ue_status check_plan(const ue_plan_buffers *p)
{
    if (!p) return fail(UE_ERR_INVALID_ARG, "plan is NULL");
    const int32_t *f[11] = {p->slot_expert, p->slot_quota, p->rep_off, p->rep_slot, p->rep_cum, p->rep_experts,
                            p->load, p->rank_off, p->rank_load_before, p->rank_load_after, p->info};
    for (int i = 0; i < 11; ++i)
        if (!f[i]) return fail(UE_ERR_INVALID_ARG, "plan array %d is NULL", i);
    return UE_OK;
}

ue_status check_ctx(const ue_ctx *ctx)
{
    if (!ctx) return fail(UE_ERR_INVALID_ARG, "context is NULL");
    return UE_OK;
}

// CTAs per simulated rank (one cluster per rank) for load / reroute: as many
// as keep the grid within one wave of two 512-thread CTAs per SM, leaving
// room for the planner's cluster that runs beside the reroute grid, with at
// least 2048 ids per CTA.
int choose_cluster(const ue::Shape &sh, int sms)
{
    const int64_t wave = 2 * (int64_t)sms - 2 * ue::kMaxCluster;
    int C = 1;
    while (C < ue::kMaxCluster && (int64_t)sh.N * C * 2 <= wave && sh.per_rank / (2 * C) >= 2048) C *= 2;
    return C;
}

ue::Launch launch_of(const ue_ctx *ctx, const ue::Shape &sh)
{
    ue::Launch ln;
    ln.sms = ctx->sms;
    ln.max_smem = (size_t)ctx->max_smem;
    ln.cluster = choose_cluster(sh, ctx->sms);
    return ln;
}

// The persistent reroute over pieces is used when a CTA's share of a rank's
// ids in the rank-per-cluster kernel is large (kClusterShareMax): that kernel
// would read the ids twice, and one CTA per rank would walk all of a rank's
// quota boundaries alone.  Pieces: about kPiecesPerCta per resident CTA,
// whole multiples of kPieceQuantum ids, within the workspace and the load
// kernel's shared memory.
ue::Pieces pieces_for(const ue_ctx *ctx, const ue::Shape &sh, const ue::Launch &ln)
{
    ue::Pieces pc{0, 0, 0, 0};
    if (sh.per_rank <= 0) return pc;
    const int64_t share = ((sh.per_rank + ln.cluster - 1) / ln.cluster + 31) / 32 * 32;
    if (share <= kClusterShareMax) return pc;
    const size_t rp_smem = ue::reroute_pieces_smem_bytes(sh);
    if (rp_smem > (size_t)ctx->max_smem) return pc;
    const int per_sm = std::min<int>(ctx->rp_blocks, ctx->smem_per_sm / (int)(rp_smem + ctx->smem_reserved));
    const int grid = ctx->sms * std::max(per_sm, 1);
    // Pieces per rank within the workspace and within the load kernel's
    // shared memory (each of its CTAs keeps its pieces' counts).
    const int64_t b_ws = (kWsInts - kWsHead) / ((int64_t)sh.N * (sh.E + 1)) - 1;
    const int64_t ppc_smem = ((int64_t)ctx->max_smem - (int64_t)ue::load_smem_bytes(sh, 0)) /
                             ((int64_t)(sh.E + 1) * (int64_t)sizeof(int32_t));
    const int64_t b_cap = std::min(b_ws, ppc_smem * ln.cluster);
    if (grid < 1 || b_cap < 1) return pc;
    int64_t B = ((int64_t)kPiecesPerCta * grid + sh.N - 1) / sh.N;
    B = std::max<int64_t>(1, std::min(B, b_cap));
    int64_t zp = ((sh.per_rank + B - 1) / B + kPieceQuantum - 1) / kPieceQuantum * kPieceQuantum;
    B = (sh.per_rank + zp - 1) / zp;
    pc.B = (int)B;
    pc.zp = zp;
    pc.NP = (int)(sh.N * B);
    pc.grid = grid;
    return pc;
}

// Run fn with ctx's device current, restoring the caller's device.
template <class F>
ue_status on_device(const ue_ctx *ctx, F &&fn)
{
    int prev = -1;
    cudaError_t e = cudaGetDevice(&prev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (prev != ctx->device && (e = cudaSetDevice(ctx->device)) != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
    ue_status s = fn();
    if (prev != ctx->device) cudaSetDevice(prev);
    return s;
}

// The context's load vector for a fused load + plan on stream st, cleared
// first when an earlier call queued a load grid without its planner; nullptr
// if that clear could not be queued.
int32_t *load_vector(ue_ctx *ctx, cudaStream_t st)
{
    int32_t *lv = ctx->ws + kWsLoadVec;
    if (ctx->lv_dirty) {
        if (cudaMemsetAsync(lv, 0, ue::kMaxE * sizeof(int32_t), st) != cudaSuccess) return nullptr;
        ctx->lv_dirty = false;
    }
    return lv;
}

}  // namespace

extern "C" {

const char *ue_status_string(ue_status s)
{
    switch (s) {
    case UE_OK: return "UE_OK";
    case UE_ERR_INVALID_ARG: return "UE_ERR_INVALID_ARG";
    case UE_ERR_CUDA: return "UE_ERR_CUDA";
    case UE_ERR_UNSUPPORTED: return "UE_ERR_UNSUPPORTED";
    case UE_ERR_DEVICE: return "UE_ERR_DEVICE";
    }
    return "UE_ERR_UNKNOWN";
}

const char *ue_last_error(void) { return g_last_error; }

ue_status ue_plan_sizes(const ue_config *cfg, int64_t sizes[11])
{
    ue::Shape sh{};
    ue_status s = make_shape(cfg, false, &sh);
    if (s != UE_OK) return s;
    if (!sizes) return fail(UE_ERR_INVALID_ARG, "sizes is NULL");
    const int64_t v[11] = {sh.S, sh.S, sh.E + 1, sh.E + sh.NR, sh.E + sh.NR, sh.E,
                           sh.E, (int64_t)sh.N * sh.E, sh.N, sh.N, 8};
    memcpy(sizes, v, sizeof v);
    return UE_OK;
}

ue_status ue_ctx_create(int device, ue_ctx **out)
{
    if (!out) return fail(UE_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    int ndev = 0;
    cudaError_t e = cudaGetDeviceCount(&ndev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceCount");
    if (device < 0 || device >= ndev) return fail(UE_ERR_INVALID_ARG, "device %d not in [0, %d)", device, ndev);
    cudaDeviceProp prop;
    if ((e = cudaGetDeviceProperties(&prop, device)) != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
    if (prop.major != 10)
        return fail(UE_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", device,
                    prop.major, prop.minor);
    ue_ctx tmp;
    tmp.device = device;
    tmp.sms = prop.multiProcessorCount;
    tmp.max_smem = (int)prop.sharedMemPerBlockOptin;
    tmp.smem_per_sm = (int)prop.sharedMemPerMultiprocessor;
    tmp.smem_reserved = (int)prop.reservedSharedMemPerBlock;
    tmp.dev_err = nullptr;
    tmp.ws = nullptr;
    tmp.wait_ns = 2000000000LL;
    tmp.stall_once = 0;
    tmp.lv_dirty = false;
    ue_status s = on_device(&tmp, [&]() -> ue_status {
        cudaError_t err;
        const size_t m = (size_t)tmp.max_smem;
        if ((err = ue::set_load_attributes(m)) != cudaSuccess) return cuda_fail(err, "load attributes");
        if ((err = ue::set_reroute_attributes(m)) != cudaSuccess) return cuda_fail(err, "reroute attributes");
        if ((err = ue::set_plan_attributes(m)) != cudaSuccess) return cuda_fail(err, "plan attributes");
        if ((err = ue::set_sync_attributes(m)) != cudaSuccess) return cuda_fail(err, "sync attributes");
        if ((err = ue::set_shard_attributes(m)) != cudaSuccess) return cuda_fail(err, "shard attributes");
        if ((err = ue::set_reroute_pieces_attributes(m)) != cudaSuccess) return cuda_fail(err, "reroute attributes");
        if ((err = ue::set_grad_bulk_attributes(m)) != cudaSuccess) return cuda_fail(err, "grad-reduce attributes");
        tmp.rp_blocks = ue::reroute_pieces_blocks_per_sm(0);
        if ((err = cudaMalloc(&tmp.dev_err, sizeof(int32_t))) != cudaSuccess) return cuda_fail(err, "cudaMalloc");
        if ((err = cudaMemset(tmp.dev_err, 0, sizeof(int32_t))) != cudaSuccess ||
            (err = cudaMalloc(&tmp.ws, kWsInts * sizeof(int32_t))) != cudaSuccess ||
            (err = cudaMemset(tmp.ws, 0, kWsHead * sizeof(int32_t))) != cudaSuccess) {
            cudaFree(tmp.dev_err);
            return cuda_fail(err, "workspace");
        }
        return UE_OK;
    });
    if (s != UE_OK) return s;
    ue_ctx *ctx = new (std::nothrow) ue_ctx(tmp);
    if (!ctx) {
        on_device(&tmp, [&]() { cudaFree(tmp.dev_err); cudaFree(tmp.ws); return UE_OK; });
        return fail(UE_ERR_INVALID_ARG, "out of host memory");
    }
    *out = ctx;
    return UE_OK;
}

ue_status ue_ctx_destroy(ue_ctx *ctx)
{
    if (!ctx) return UE_OK;
    ue_status s = on_device(ctx, [&]() -> ue_status {
        cudaError_t e = cudaFree(ctx->dev_err);
        const cudaError_t e2 = cudaFree(ctx->ws);
        if (e == cudaSuccess) e = e2;
        return e == cudaSuccess ? UE_OK : cuda_fail(e, "cudaFree");
    });
    delete ctx;
    return s;
}

ue_status ue_ctx_set_wait_limit(ue_ctx *ctx, int64_t limit_ns, int32_t flags)
{
    ue_status s = check_ctx(ctx);
    if (s != UE_OK) return s;
    if (limit_ns < 1000 || limit_ns > 60000000000LL)
        return fail(UE_ERR_INVALID_ARG, "limit_ns=%lld outside [1000, 6e10]", (long long)limit_ns);
    if (flags & ~UE_WAIT_STALL_ONCE) return fail(UE_ERR_INVALID_ARG, "flags=%d (bit 0: UE_WAIT_STALL_ONCE)", flags);
    ctx->wait_ns = limit_ns;
    ctx->stall_once = (flags & UE_WAIT_STALL_ONCE) ? 1 : 0;
    return UE_OK;
}

ue_status ue_ctx_device_error(ue_ctx *ctx, int32_t *host_word, void *stream)
{
    ue_status s = check_ctx(ctx);
    if (s != UE_OK) return s;
    if (!host_word) return fail(UE_ERR_INVALID_ARG, "host_word is NULL");
    return on_device(ctx, [&]() -> ue_status {
        cudaStream_t st = static_cast<cudaStream_t>(stream);
        cudaError_t e = cudaMemcpyAsync(host_word, ctx->dev_err, sizeof(int32_t), cudaMemcpyDeviceToHost, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e == cudaSuccess) e = cudaMemsetAsync(ctx->dev_err, 0, sizeof(int32_t), st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        return e == cudaSuccess ? UE_OK : cuda_fail(e, "device status word");
    });
}

ue_status ue_load(ue_ctx *ctx, const ue_config *cfg, const int32_t *ids, int32_t *counts, int32_t *bad,
                  void *stream)
{
    ue::Shape sh{};
    ue_status s = make_shape(cfg, true, &sh);
    if (s != UE_OK) return s;
    if (!counts) return fail(UE_ERR_INVALID_ARG, "counts is NULL");
    if (sh.T > 0 && (!ids || !aligned16(ids))) return fail(UE_ERR_INVALID_ARG, "ids must be non-NULL and 16-byte aligned");
    if ((s = check_ctx(ctx)) != UE_OK) return s;
    return on_device(ctx, [&]() -> ue_status {
        cudaError_t e = ue::launch_load(sh, launch_of(ctx, sh), ids, counts, bad, static_cast<cudaStream_t>(stream));
        return e == cudaSuccess ? UE_OK : cuda_fail(e, "load launch");
    });
}

ue_status ue_plan_ex(ue_ctx *ctx, const ue_config *cfg, const int32_t *counts, const ue_plan_buffers *plan,
                     int variant, void *stream)
{
    ue::Shape sh{};
    ue_status s = make_shape(cfg, false, &sh);
    if (s == UE_OK) s = check_plan(plan);
    if (s != UE_OK) return s;
    if (variant < 0 || variant > (UE_PLAN_REQUEUE | UE_PLAN_SPREAD))
        return fail(UE_ERR_INVALID_ARG, "variant=%d (bits: 1 requeue, 2 spread)", variant);
    if (!counts) return fail(UE_ERR_INVALID_ARG, "counts is NULL");
    if ((s = check_ctx(ctx)) != UE_OK) return s;
    if (ue::plan_smem_bytes(sh) > (size_t)ctx->max_smem)
        return fail(UE_ERR_INVALID_ARG, "plan needs %zu bytes of shared memory (> %d)", ue::plan_smem_bytes(sh),
                    ctx->max_smem);
    return on_device(ctx, [&]() -> ue_status {
        cudaError_t e = ue::launch_plan(sh, counts, ue::to_dev(*plan), static_cast<cudaStream_t>(stream), false,
                                        variant);
        return e == cudaSuccess ? UE_OK : cuda_fail(e, "plan launch");
    });
}

ue_status ue_plan(ue_ctx *ctx, const ue_config *cfg, const int32_t *counts, const ue_plan_buffers *plan,
                  void *stream)
{
    return ue_plan_ex(ctx, cfg, counts, plan, 0, stream);
}

ue_status ue_reroute(ue_ctx *ctx, const ue_config *cfg, const int32_t *ids, const ue_plan_buffers *plan,
                     int32_t *phys, void *stream)
{
    ue::Shape sh{};
    ue_status s = make_shape(cfg, true, &sh);
    if (s == UE_OK) s = check_plan(plan);
    if (s != UE_OK) return s;
    if (sh.T > 0 && (!ids || !aligned16(ids))) return fail(UE_ERR_INVALID_ARG, "ids must be non-NULL and 16-byte aligned");
    if (sh.T > 0 && !phys) return fail(UE_ERR_INVALID_ARG, "phys is NULL");
    if ((s = check_ctx(ctx)) != UE_OK) return s;
    if (ue::reroute_smem_bytes(sh, false, 0, false) > (size_t)ctx->max_smem)
        return fail(UE_ERR_INVALID_ARG, "reroute needs %zu bytes of shared memory (> %d)",
                    ue::reroute_smem_bytes(sh, false, 0, false), ctx->max_smem);
    return on_device(ctx, [&]() -> ue_status {
        const cudaStream_t st = static_cast<cudaStream_t>(stream);
        const ue::Launch ln = launch_of(ctx, sh);
        const ue::Pieces pc = pieces_for(ctx, sh, ln);
        cudaError_t e;
        if (pc.NP > 0) {
            // The piece rows first (no counts), then the persistent reroute.
            if ((e = ue::launch_load(sh, ln, ids, nullptr, nullptr, st, &pc, ctx->ws + kWsHead)) != cudaSuccess)
                return cuda_fail(e, "load launch");
            e = ue::launch_reroute_pieces(sh, pc, ids, ue::to_dev(*plan), ctx->ws + kWsHead, ctx->ws, phys, st,
                                          false);
        } else {
            e = ue::launch_reroute(sh, ln, ids, ue::to_dev(*plan), phys, st, false);
        }
        return e == cudaSuccess ? UE_OK : cuda_fail(e, "reroute launch");
    });
}

ue_status ue_rebalance_ex(ue_ctx *ctx, const ue_config *cfg, const int32_t *ids, int32_t *counts, int32_t *bad,
                          const ue_plan_buffers *plan, int32_t *phys, int variant, void *stream)
{
    // Validate everything before the first launch so a refusal leaves all outputs untouched.
    ue::Shape sh{};
    ue_status s = make_shape(cfg, true, &sh);
    if (s == UE_OK) s = check_plan(plan);
    if (s != UE_OK) return s;
    if (variant < 0 || variant > (UE_PLAN_REQUEUE | UE_PLAN_SPREAD))
        return fail(UE_ERR_INVALID_ARG, "variant=%d (bits: 1 requeue, 2 spread)", variant);
    if (!counts) return fail(UE_ERR_INVALID_ARG, "counts is NULL");
    if (sh.T > 0 && (!ids || !aligned16(ids))) return fail(UE_ERR_INVALID_ARG, "ids must be non-NULL and 16-byte aligned");
    if (sh.T > 0 && !phys) return fail(UE_ERR_INVALID_ARG, "phys is NULL");
    if ((s = check_ctx(ctx)) != UE_OK) return s;
    if (ue::plan_smem_bytes(sh) > (size_t)ctx->max_smem || ue::reroute_smem_bytes(sh, false, 0, false) > (size_t)ctx->max_smem)
        return fail(UE_ERR_INVALID_ARG, "shape needs more shared memory than the device offers");
    return on_device(ctx, [&]() -> ue_status {
        const cudaStream_t st = static_cast<cudaStream_t>(stream);
        const ue::Launch ln = launch_of(ctx, sh);
        const ue::PlanDev pd = ue::to_dev(*plan);
        const ue::Pieces pc = pieces_for(ctx, sh, ln);
        int32_t *lv = load_vector(ctx, st);
        if (lv == nullptr) return cuda_fail(cudaGetLastError(), "load vector reset");
        cudaError_t e = ue::launch_load(sh, ln, ids, counts, bad, st, &pc, ctx->ws + kWsHead, lv);
        if (e != cudaSuccess) return cuda_fail(e, "load launch");
        // The planner and the reroute kernel use programmatic dependent launch:
        // each may start while its predecessor drains, and waits for it
        // (griddepcontrol.wait) before reading what it wrote.
        if ((e = ue::launch_plan(sh, counts, pd, st, true, variant, lv)) != cudaSuccess) {
            ctx->lv_dirty = true;
            return cuda_fail(e, "plan launch");
        }
        e = pc.NP > 0 ? ue::launch_reroute_pieces(sh, pc, ids, pd, ctx->ws + kWsHead, ctx->ws, phys, st, true)
                      : ue::launch_reroute(sh, ln, ids, pd, phys, st, true);
        if (e != cudaSuccess) return cuda_fail(e, "reroute launch");
        return UE_OK;
    });
}

ue_status ue_rebalance(ue_ctx *ctx, const ue_config *cfg, const int32_t *ids, int32_t *counts, int32_t *bad,
                       const ue_plan_buffers *plan, int32_t *phys, void *stream)
{
    return ue_rebalance_ex(ctx, cfg, ids, counts, bad, plan, phys, 0, stream);
}

namespace {
ue_status check_dispatch(const ue::Shape &sh, const ue_dispatch_buffers *d, ue::DispatchOut *out)
{
    if (!d) return fail(UE_ERR_INVALID_ARG, "dispatch buffers are NULL");
    if (!d->slot_off) return fail(UE_ERR_INVALID_ARG, "slot_off is NULL");
    if (sh.T > 0 && !d->src_index) return fail(UE_ERR_INVALID_ARG, "src_index is NULL");
    if (sh.T > 0 && d->gates && !d->gates_out) return fail(UE_ERR_INVALID_ARG, "gates given but gates_out is NULL");
    out->gates = sh.T > 0 ? d->gates : nullptr;
    out->slot_off = d->slot_off;
    out->src_index = d->src_index;
    out->gates_out = d->gates_out;
    return UE_OK;
}
}  // namespace

ue_status ue_dispatch(ue_ctx *ctx, const ue_config *cfg, const int32_t *ids, const ue_plan_buffers *plan,
                      int32_t *phys, const ue_dispatch_buffers *disp, void *stream)
{
    ue::Shape sh{};
    ue::DispatchOut out{};
    ue_status s = make_shape(cfg, true, &sh);
    if (s == UE_OK) s = check_plan(plan);
    if (s == UE_OK) s = check_dispatch(sh, disp, &out);
    if (s != UE_OK) return s;
    if (sh.T > 0 && (!ids || !aligned16(ids))) return fail(UE_ERR_INVALID_ARG, "ids must be non-NULL and 16-byte aligned");
    if (sh.T > 0 && !phys) return fail(UE_ERR_INVALID_ARG, "phys is NULL");
    if ((s = check_ctx(ctx)) != UE_OK) return s;
    if (ue::reroute_smem_bytes(sh, true, 0, false) > (size_t)ctx->max_smem)
        return fail(UE_ERR_INVALID_ARG, "dispatch needs %zu bytes of shared memory (> %d)",
                    ue::reroute_smem_bytes(sh, true, 0, false), ctx->max_smem);
    return on_device(ctx, [&]() -> ue_status {
        cudaError_t e = ue::launch_dispatch(sh, launch_of(ctx, sh), ids, ue::to_dev(*plan), phys, out, ctx->dev_err,
                                            static_cast<cudaStream_t>(stream), false);
        return e == cudaSuccess ? UE_OK : cuda_fail(e, "dispatch launch");
    });
}

ue_status ue_rebalance_dispatch(ue_ctx *ctx, const ue_config *cfg, const int32_t *ids, int32_t *counts,
                                int32_t *bad, const ue_plan_buffers *plan, int32_t *phys,
                                const ue_dispatch_buffers *disp, void *stream)
{
    ue::Shape sh{};
    ue::DispatchOut out{};
    ue_status s = make_shape(cfg, true, &sh);
    if (s == UE_OK) s = check_plan(plan);
    if (s == UE_OK) s = check_dispatch(sh, disp, &out);
    if (s != UE_OK) return s;
    if (!counts) return fail(UE_ERR_INVALID_ARG, "counts is NULL");
    if (sh.T > 0 && (!ids || !aligned16(ids))) return fail(UE_ERR_INVALID_ARG, "ids must be non-NULL and 16-byte aligned");
    if (sh.T > 0 && !phys) return fail(UE_ERR_INVALID_ARG, "phys is NULL");
    if ((s = check_ctx(ctx)) != UE_OK) return s;
    if (ue::plan_smem_bytes(sh) > (size_t)ctx->max_smem || ue::reroute_smem_bytes(sh, true, 0, false) > (size_t)ctx->max_smem)
        return fail(UE_ERR_INVALID_ARG, "shape needs more shared memory than the device offers");
    return on_device(ctx, [&]() -> ue_status {
        const cudaStream_t st = static_cast<cudaStream_t>(stream);
        const ue::Launch ln = launch_of(ctx, sh);
        const ue::PlanDev pd = ue::to_dev(*plan);
        int32_t *lv = load_vector(ctx, st);
        if (lv == nullptr) return cuda_fail(cudaGetLastError(), "load vector reset");
        cudaError_t e = ue::launch_load(sh, ln, ids, counts, bad, st, nullptr, nullptr, lv);
        if (e != cudaSuccess) return cuda_fail(e, "load launch");
        if ((e = ue::launch_plan(sh, counts, pd, st, true, 0, lv)) != cudaSuccess) {
            ctx->lv_dirty = true;
            return cuda_fail(e, "plan launch");
        }
        if ((e = ue::launch_dispatch(sh, ln, ids, pd, phys, out, ctx->dev_err, st, true)) != cudaSuccess)
            return cuda_fail(e, "dispatch launch");
        return UE_OK;
    });
}

namespace {
ue_status sync_common(ue_ctx *ctx, const ue_config *cfg, void *weights, int64_t slot_bytes,
                      const ue_plan_buffers *plan, const int32_t *prev, void *stream)
{
    ue::Shape sh{};
    ue_status s = make_shape(cfg, false, &sh);
    if (s == UE_OK) s = check_plan(plan);
    if (s != UE_OK) return s;
    if (!weights || !aligned16(weights)) return fail(UE_ERR_INVALID_ARG, "weights must be non-NULL and 16-byte aligned");
    if (slot_bytes <= 0 || slot_bytes % 16 != 0)
        return fail(UE_ERR_INVALID_ARG, "slot_bytes=%lld must be a positive multiple of 16", (long long)slot_bytes);
    if ((s = check_ctx(ctx)) != UE_OK) return s;
    if (ue::sync_smem_bytes(sh) > (size_t)ctx->max_smem)
        return fail(UE_ERR_INVALID_ARG, "sync needs %zu bytes of shared memory (> %d)", ue::sync_smem_bytes(sh),
                    ctx->max_smem);
    return on_device(ctx, [&]() -> ue_status {
        const ue::WaitBound wb{(unsigned long long)ctx->wait_ns, ctx->stall_once};
        cudaError_t e = ue::launch_sync(sh, launch_of(ctx, sh), static_cast<uint8_t *>(weights), slot_bytes,
                                        ue::to_dev(*plan), prev, ctx->dev_err, static_cast<cudaStream_t>(stream), wb);
        ctx->stall_once = 0;
        return e == cudaSuccess ? UE_OK : cuda_fail(e, "sync launch");
    });
}
}  // namespace

ue_status ue_sync(ue_ctx *ctx, const ue_config *cfg, void *weights, int64_t slot_bytes, const ue_plan_buffers *plan,
                  void *stream)
{
    return sync_common(ctx, cfg, weights, slot_bytes, plan, nullptr, stream);
}

ue_status ue_sync_delta(ue_ctx *ctx, const ue_config *cfg, void *weights, int64_t slot_bytes,
                        const ue_plan_buffers *plan, const int32_t *prev_slot_expert, void *stream)
{
    return sync_common(ctx, cfg, weights, slot_bytes, plan, prev_slot_expert, stream);
}

ue_status ue_sync_restore(ue_ctx *ctx, const ue_config *cfg, void *weights, int64_t slot_bytes,
                          const ue_plan_buffers *plan, const int32_t *held_slot_expert, void *stream)
{
    // The incremental sync towards the saved plan: every filled redundant slot
    // whose expert differs from the one it holds now receives its home slot.
    return sync_common(ctx, cfg, weights, slot_bytes, plan, held_slot_expert, stream);
}

ue_status ue_grad_reduce(ue_ctx *ctx, const ue_config *cfg, float *master, const void *grads, int grad_dtype,
                         int64_t P, const ue_plan_buffers *plan, void *stream)
{
    ue::Shape sh{};
    ue_status s = make_shape(cfg, false, &sh);
    if (s == UE_OK) s = check_plan(plan);
    if (s != UE_OK) return s;
    if (grad_dtype != 0 && grad_dtype != 1) return fail(UE_ERR_INVALID_ARG, "grad_dtype=%d (0 = fp32, 1 = bf16)", grad_dtype);
    if (P <= 0 || P % 8 != 0) return fail(UE_ERR_INVALID_ARG, "P=%lld must be a positive multiple of 8", (long long)P);
    if (!master || !aligned16(master)) return fail(UE_ERR_INVALID_ARG, "master must be non-NULL and 16-byte aligned");
    if (sh.NR > 0 && (!grads || !aligned16(grads)))
        return fail(UE_ERR_INVALID_ARG, "grads must be non-NULL and 16-byte aligned");
    if ((s = check_ctx(ctx)) != UE_OK) return s;
    return on_device(ctx, [&]() -> ue_status {
        cudaError_t e;
        if (ue::grad_bulk_smem_bytes(sh) <= (size_t)ctx->max_smem) {
            const ue::WaitBound wb{(unsigned long long)ctx->wait_ns, ctx->stall_once};
            e = ue::launch_grad_reduce_bulk(sh, ctx->sms, master, grads, grad_dtype, P, ue::to_dev(*plan),
                                            ctx->dev_err, static_cast<cudaStream_t>(stream), wb);
            ctx->stall_once = 0;
        } else {
            const ue::Launch ln = launch_of(ctx, sh);
            e = ue::launch_grad_reduce(sh, ln, master, grads, grad_dtype, P, ue::to_dev(*plan),
                                       static_cast<cudaStream_t>(stream));
        }
        return e == cudaSuccess ? UE_OK : cuda_fail(e, "grad-reduce launch");
    });
}

// ---- calls across GPUs ---------------------------------------------------------

namespace {
ue_status check_shard(const ue::Shape &sh, const ue_shard *shard)
{
    if (!shard) return fail(UE_ERR_INVALID_ARG, "shard is NULL");
    if (shard->G < 1 || shard->G > ue::kMaxGpus)
        return fail(UE_ERR_INVALID_ARG, "G=%d outside [1, %d]", shard->G, ue::kMaxGpus);
    if (sh.N % shard->G != 0) return fail(UE_ERR_INVALID_ARG, "N=%d is not a multiple of G=%d", sh.N, shard->G);
    if (shard->g < 0 || shard->g >= shard->G) return fail(UE_ERR_INVALID_ARG, "g=%d not in [0, %d)", shard->g, shard->G);
    return UE_OK;
}

// The shape of this GPU's ranks for the rank-per-cluster kernels: N / G ranks
// and their tokens; everything that indexes slots or experts stays global.
ue::Shape local_shape(const ue::Shape &sh, const ue_shard *shard)
{
    ue::Shape l = sh;
    l.N = sh.N / shard->G;
    l.T = sh.T / shard->G;
    return l;
}

ue_status peer_table(const void *const *bases, int G, ue::PeerTable *t, const char *what)
{
    if (!bases) return fail(UE_ERR_INVALID_ARG, "%s is NULL", what);
    for (int h = 0; h < ue::kMaxGpus; ++h) t->p[h] = nullptr;
    for (int h = 0; h < G; ++h) {
        if (!bases[h] || !aligned16(bases[h]))
            return fail(UE_ERR_INVALID_ARG, "%s[%d] must be non-NULL and 16-byte aligned", what, h);
        t->p[h] = bases[h];
    }
    return UE_OK;
}
}  // namespace

int32_t ue_relay_rounds(int32_t G) { return G < 1 || G > ue::kMaxGpus ? -1 : ue::relay_rounds(G); }

ue_status ue_load_shard(ue_ctx *ctx, const ue_config *cfg, const ue_shard *shard, const int32_t *ids_local,
                        int32_t *counts, int32_t *bad, void *stream)
{
    ue::Shape sh{};
    ue_status s = make_shape(cfg, true, &sh);
    if (s == UE_OK) s = check_shard(sh, shard);
    if (s != UE_OK) return s;
    if (!counts) return fail(UE_ERR_INVALID_ARG, "counts is NULL");
    const ue::Shape l = local_shape(sh, shard);
    if (l.T > 0 && (!ids_local || !aligned16(ids_local)))
        return fail(UE_ERR_INVALID_ARG, "ids_local must be non-NULL and 16-byte aligned");
    if ((s = check_ctx(ctx)) != UE_OK) return s;
    const int64_t r0 = (int64_t)shard->g * l.N;
    return on_device(ctx, [&]() -> ue_status {
        cudaError_t e = ue::launch_load(l, launch_of(ctx, l), ids_local, counts + r0 * sh.E, bad ? bad + r0 : nullptr,
                                        static_cast<cudaStream_t>(stream));
        return e == cudaSuccess ? UE_OK : cuda_fail(e, "load launch");
    });
}

ue_status ue_reroute_shard(ue_ctx *ctx, const ue_config *cfg, const ue_shard *shard, const int32_t *ids_local,
                           const ue_plan_buffers *plan, int32_t *phys_local, void *stream)
{
    ue::Shape sh{};
    ue_status s = make_shape(cfg, true, &sh);
    if (s == UE_OK) s = check_shard(sh, shard);
    if (s == UE_OK) s = check_plan(plan);
    if (s != UE_OK) return s;
    const ue::Shape l = local_shape(sh, shard);
    if (l.T > 0 && (!ids_local || !aligned16(ids_local)))
        return fail(UE_ERR_INVALID_ARG, "ids_local must be non-NULL and 16-byte aligned");
    if (l.T > 0 && !phys_local) return fail(UE_ERR_INVALID_ARG, "phys_local is NULL");
    if ((s = check_ctx(ctx)) != UE_OK) return s;
    if (ue::reroute_smem_bytes(l, false, 0, false) > (size_t)ctx->max_smem)
        return fail(UE_ERR_INVALID_ARG, "reroute needs %zu bytes of shared memory (> %d)",
                    ue::reroute_smem_bytes(l, false, 0, false), ctx->max_smem);
    ue::PlanDev pd = ue::to_dev(*plan);
    pd.rank_off += (int64_t)shard->g * l.N * sh.E;     // this GPU's rows of rank_off
    return on_device(ctx, [&]() -> ue_status {
        const cudaStream_t st = static_cast<cudaStream_t>(stream);
        const ue::Launch ln = launch_of(ctx, l);
        const ue::Pieces pc = pieces_for(ctx, l, ln);
        cudaError_t e;
        if (pc.NP > 0) {
            if ((e = ue::launch_load(l, ln, ids_local, nullptr, nullptr, st, &pc, ctx->ws + kWsHead)) != cudaSuccess)
                return cuda_fail(e, "load launch");
            e = ue::launch_reroute_pieces(l, pc, ids_local, pd, ctx->ws + kWsHead, ctx->ws, phys_local, st, false);
        } else {
            e = ue::launch_reroute(l, ln, ids_local, pd, phys_local, st, false);
        }
        return e == cudaSuccess ? UE_OK : cuda_fail(e, "reroute launch");
    });
}

ue_status ue_sync_shard(ue_ctx *ctx, const ue_config *cfg, const ue_shard *shard, void *const *slot_bases,
                        int64_t slot_bytes, const ue_plan_buffers *plan, int32_t round, void *stream)
{
    ue::Shape sh{};
    ue_status s = make_shape(cfg, false, &sh);
    if (s == UE_OK) s = check_shard(sh, shard);
    if (s == UE_OK) s = check_plan(plan);
    if (s != UE_OK) return s;
    ue::PeerTable t;
    if ((s = peer_table(const_cast<const void *const *>(slot_bases), shard->G, &t, "slot_bases")) != UE_OK) return s;
    if (slot_bytes <= 0 || slot_bytes % 16 != 0)
        return fail(UE_ERR_INVALID_ARG, "slot_bytes=%lld must be a positive multiple of 16", (long long)slot_bytes);
    if (round < -1 || round >= ue::relay_rounds(shard->G))
        return fail(UE_ERR_INVALID_ARG, "round=%d not in [-1, %d)", round, ue::relay_rounds(shard->G));
    if ((s = check_ctx(ctx)) != UE_OK) return s;
    if (ue::sync_shard_smem_bytes(sh) > (size_t)ctx->max_smem)
        return fail(UE_ERR_INVALID_ARG, "sync needs %zu bytes of shared memory (> %d)", ue::sync_shard_smem_bytes(sh),
                    ctx->max_smem);
    return on_device(ctx, [&]() -> ue_status {
        const ue::WaitBound wb{(unsigned long long)ctx->wait_ns, ctx->stall_once};
        cudaError_t e = ue::launch_sync_shard(sh, launch_of(ctx, sh), t, static_cast<uint8_t *>(slot_bases[shard->g]),
                                              shard->G, shard->g, round, slot_bytes, ue::to_dev(*plan), ctx->dev_err,
                                              static_cast<cudaStream_t>(stream), wb);
        ctx->stall_once = 0;
        return e == cudaSuccess ? UE_OK : cuda_fail(e, "sync launch");
    });
}

ue_status ue_grad_reduce_shard(ue_ctx *ctx, const ue_config *cfg, const ue_shard *shard, float *master_local,
                               const void *const *grad_bases, int grad_dtype, int64_t P,
                               const ue_plan_buffers *plan, void *stream)
{
    ue::Shape sh{};
    ue_status s = make_shape(cfg, false, &sh);
    if (s == UE_OK) s = check_shard(sh, shard);
    if (s == UE_OK) s = check_plan(plan);
    if (s != UE_OK) return s;
    if (grad_dtype != 0 && grad_dtype != 1) return fail(UE_ERR_INVALID_ARG, "grad_dtype=%d (0 = fp32, 1 = bf16)", grad_dtype);
    if (P <= 0 || P % 8 != 0) return fail(UE_ERR_INVALID_ARG, "P=%lld must be a positive multiple of 8", (long long)P);
    if (!master_local || !aligned16(master_local))
        return fail(UE_ERR_INVALID_ARG, "master_local must be non-NULL and 16-byte aligned");
    ue::PeerTable t;
    if (sh.NR > 0) {
        if ((s = peer_table(grad_bases, shard->G, &t, "grad_bases")) != UE_OK) return s;
    } else {
        for (int h = 0; h < ue::kMaxGpus; ++h) t.p[h] = nullptr;
    }
    if ((s = check_ctx(ctx)) != UE_OK) return s;
    return on_device(ctx, [&]() -> ue_status {
        if (ue::grad_bulk_smem_bytes(sh) <= (size_t)ctx->max_smem) {
            const ue::WaitBound wb{(unsigned long long)ctx->wait_ns, ctx->stall_once};
            cudaError_t e = ue::launch_grad_reduce_bulk_shard(sh, ctx->sms, master_local, t, shard->G, shard->g,
                                                              grad_dtype, P, ue::to_dev(*plan), ctx->dev_err,
                                                              static_cast<cudaStream_t>(stream), wb);
            ctx->stall_once = 0;
            return e == cudaSuccess ? UE_OK : cuda_fail(e, "grad-reduce launch");
        }
        const ue::Launch ln = launch_of(ctx, sh);
        cudaError_t e = ue::launch_grad_reduce_shard(sh, ln, master_local, t, shard->G, shard->g, grad_dtype, P,
                                                     ue::to_dev(*plan), static_cast<cudaStream_t>(stream));
        return e == cudaSuccess ? UE_OK : cuda_fail(e, "grad-reduce launch");
    });
}

}  // extern "C"

// ---- routing expansion without a context ------------------------------------------
//
// Some callers cannot call cudaMalloc: an engine that reserves its whole
// device-memory budget in its own pool at start-up (an allocation outside the
// pool fails or breaks its accounting), or a caller inside a region of its
// framework where allocation is not allowed.  Such a caller cannot create a
// ue_ctx, which allocates its status word and workspace.  ue_reroute_static
// runs the reroute over pieces (the load kernel's piece pass, then the
// persistent reroute kernel) with its scratch - the piece counters and the rows
// of occurrences before each piece - in g_scratch, a device array the library
// holds on every GPU that loads it until the process exits.  The caller passes
// ids, the plan and phys as for ue_reroute and gets the same phys.
//
// In host code g_scratch names a host-side stand-in for the device symbol:
// the first call on each device, with that device current, asks the runtime
// for its device address (cudaGetSymbolAddress) and sets the kernels'
// shared-memory limits; later calls on that device reuse them.

namespace {

constexpr int64_t kStaticScratchInts = (int64_t)1 << 20;   // 4 MiB
constexpr int64_t kStaticHead = 64;                          // the piece counters, then the rows
constexpr int kStaticMaxDevices = 64;

static __device__ __align__(256) int32_t g_scratch[kStaticScratchInts];

struct StaticSetup {
    bool ready;
    int32_t *scratch;      // g_scratch's address on the device
    ue_ctx props;          // device properties (sms, shared memory, resident CTAs); no allocations
};
StaticSetup g_static[kStaticMaxDevices];
std::mutex g_static_lock;

}  // namespace

extern "C" ue_status ue_reroute_static(const ue_config *cfg, const int32_t *ids, const ue_plan_buffers *plan,
                                       int32_t *phys, void *stream)
{
    ue::Shape sh{};
    ue_status s = make_shape(cfg, true, &sh);
    if (s == UE_OK) s = check_plan(plan);
    if (s != UE_OK) return s;
    if (sh.T > 0 && (!ids || !aligned16(ids))) return fail(UE_ERR_INVALID_ARG, "ids must be non-NULL and 16-byte aligned");
    if (sh.T > 0 && !phys) return fail(UE_ERR_INVALID_ARG, "phys is NULL");
    // At least two pieces' rows per rank must fit the static scratch.
    const int64_t row_ints = (int64_t)sh.N * (sh.E + 1);
    if (kStaticHead + 2 * row_ints > kStaticScratchInts)
        return fail(UE_ERR_INVALID_ARG,
                    "N * (E + 1) = %lld exceeds the static scratch (2 * N * (E + 1) + %lld <= %lld ints)",
                    (long long)row_ints, (long long)kStaticHead, (long long)kStaticScratchInts);
    if (sh.per_rank == 0) return UE_OK;

    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kStaticMaxDevices) return fail(UE_ERR_UNSUPPORTED, "device %d beyond %d", dev, kStaticMaxDevices);
    StaticSetup ds;
    {
        std::lock_guard<std::mutex> lock(g_static_lock);
        StaticSetup &d = g_static[dev];
        if (!d.ready) {
            cudaDeviceProp prop;
            if ((e = cudaGetDeviceProperties(&prop, dev)) != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
            if (prop.major != 10)
                return fail(UE_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", dev,
                            prop.major, prop.minor);
            void *p = nullptr;
            if ((e = cudaGetSymbolAddress(&p, g_scratch)) != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
            const size_t m = (size_t)prop.sharedMemPerBlockOptin;
            if ((e = ue::set_load_attributes(m)) != cudaSuccess) return cuda_fail(e, "load attributes");
            if ((e = ue::set_reroute_pieces_attributes(m)) != cudaSuccess) return cuda_fail(e, "reroute attributes");
            d.scratch = static_cast<int32_t *>(p);
            d.props = ue_ctx{};
            d.props.device = dev;
            d.props.sms = prop.multiProcessorCount;
            d.props.max_smem = (int)m;
            d.props.smem_per_sm = (int)prop.sharedMemPerMultiprocessor;
            d.props.smem_reserved = (int)prop.reservedSharedMemPerBlock;
            d.props.rp_blocks = ue::reroute_pieces_blocks_per_sm(0);
            d.ready = true;
        }
        ds = d;
    }

    // Pieces as for the context's workspace, within the static scratch; this
    // call takes the persistent reroute whatever the shape.
    const ue_ctx &px = ds.props;
    const ue::Launch ln = launch_of(&px, sh);
    const size_t rp_smem = ue::reroute_pieces_smem_bytes(sh);
    if (rp_smem > (size_t)px.max_smem) return fail(UE_ERR_INVALID_ARG, "E=%d too large for the reroute's tables", sh.E);
    const int per_sm = std::min<int>(px.rp_blocks, px.smem_per_sm / (int)(rp_smem + px.smem_reserved));
    ue::Pieces pc{};
    pc.grid = px.sms * std::max(per_sm, 1);
    const int64_t b_ws = (kStaticScratchInts - kStaticHead) / row_ints - 1;
    const int64_t ppc_smem = ((int64_t)px.max_smem - (int64_t)ue::load_smem_bytes(sh, 0)) /
                             ((int64_t)(sh.E + 1) * (int64_t)sizeof(int32_t));
    int64_t B = ((int64_t)kPiecesPerCta * pc.grid + sh.N - 1) / sh.N;
    B = std::max<int64_t>(1, std::min(B, std::min(b_ws, ppc_smem * ln.cluster)));
    pc.zp = ((sh.per_rank + B - 1) / B + kPieceQuantum - 1) / kPieceQuantum * kPieceQuantum;
    pc.B = (int)((sh.per_rank + pc.zp - 1) / pc.zp);
    pc.NP = sh.N * pc.B;

    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    const ue::PlanDev pd = ue::to_dev(*plan);
    // The piece counters must start at 0: the reroute kernel leaves them at 0,
    // but a call that did not complete would not have.
    if ((e = cudaMemsetAsync(ds.scratch, 0, 2 * sizeof(int32_t), st)) != cudaSuccess) return cuda_fail(e, "counters");
    if ((e = ue::launch_load(sh, ln, ids, nullptr, nullptr, st, &pc, ds.scratch + kStaticHead)) != cudaSuccess)
        return cuda_fail(e, "load launch");
    if ((e = ue::launch_reroute_pieces(sh, pc, ids, pd, ds.scratch + kStaticHead, ds.scratch, phys, st, false)) !=
        cudaSuccess)
        return cuda_fail(e, "reroute launch");
    return UE_OK;
}
