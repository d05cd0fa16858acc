// coli_moe.cu -- host side of the C ABI declared in include/coli_moe.h.
//
// Validates arguments, owns the per-handle device workspace, and enqueues the
// kernels of quant.cuh, route.cuh and expert.cuh on the caller's stream.
// No call synchronises the host except coli_moe_forward_host.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "coli_moe.h"
#include "common.cuh"
#include "expert.cuh"
#include "grouped_tc.cuh"
#include "quant.cuh"
#include "route.cuh"

using namespace coli;

namespace {

thread_local std::string g_last_error;
std::atomic<uint64_t> g_launches{0};

coli_status fail(coli_status s, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

coli_status cuda_fail(cudaError_t e, const char *what) {
    cudaGetLastError();  // clear the sticky-free error state of the runtime
    return fail(e == cudaErrorMemoryAllocation ? COLI_ENOMEM : COLI_ECUDA, "%s: %s", what,
                cudaGetErrorString(e));
}

#define COLI_CUDA(call, what)                          \
    do {                                               \
        cudaError_t e_ = (call);                       \
        if (e_ != cudaSuccess) return cuda_fail(e_, what); \
    } while (0)

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
    return n > 0 ? n : 148;
}

constexpr int MAX_SMEM = 227 * 1024;
constexpr int SMALL_T = 8;  // the few-token down+combine path handles T <= SMALL_T

// Vectors per lane template choice for a row of V uint4 vectors.
int pick_vpl(int V) {
    int need = (V + 31) / 32;
    if (need <= 1) return 1;
    if (need <= 2) return 2;
    if (need <= 4) return 4;
    if (need <= 6) return 6;
    if (need <= 12) return 12;
    return 0;  // generic loop
}

struct KernelTimer {
    const char *name;
    cudaEvent_t a, b;
};

}  // namespace

// ---------------------------------------------------------------------------
struct coli_moe {
    coli_moe_config cfg;
    const float *router_w = nullptr, *bias = nullptr;
    int device = 0, nsm = 148;
    void *ws_base = nullptr;
    size_t ws_bytes = 0;
    RouteWs rw{};
    ExpertDev *experts_dev = nullptr;
    int8_t *xq = nullptr;
    float *xd = nullptr;
    int8_t *hq = nullptr;
    float *hd = nullptr;
    float *e_pairs = nullptr;  // only when max_tokens > SMALL_T
    bool no_tc = false;        // COLI_NO_TC=1: CUDA-core grouped kernels instead (comparison runs)
    int8_t *xg = nullptr;      // x codes / scales in pair order (tensor-core path)
    float *xdg = nullptr;
    CUtensorMap *maps_dev = nullptr;  // activation maps, then gate/up/down of every expert
    double *corr_x = nullptr, *corr_h = nullptr;  // per-pair weight-offset shares
    bool tc_maps = false;
    float *x_in = nullptr, *y_out = nullptr;
    uint8_t *xrec = nullptr, *hrec = nullptr;
    int *err = nullptr;
    unsigned long long *gbar = nullptr;
    int *hcnt = nullptr;  // per active expert: gate/up items done (decode kernel)
    long long *wait_limit = nullptr;  // SM cycles a kernel's wait on progress may last
    double *out_partial = nullptr;    // set during coli_moe_forward_partial
    int last_T = 0;
    std::map<const void *, int> occ_cache;  // kernel -> CTAs per SM (attributes already set)
    // profiling
    bool profiling = false;
    std::vector<KernelTimer> pending;
    std::vector<cudaEvent_t> event_pool;
};

namespace {

struct Layout {
    size_t total = 0;
    size_t add(size_t bytes) {
        size_t off = (total + 255) & ~(size_t)255;
        total = off + bytes;
        return off;
    }
};

struct WsOffsets {
    size_t s, c, idx, w, bitmap, prefix, counter, n_active, active, off, act_of, pair_tok,
        pair_slot, tok_pair, xq, xd, hq, hd, e_pairs, xg, xdg, maps, corr_x, corr_h, x_in, y_out, experts,
        xrec, hrec,
        err, gbar, hcnt, wait_limit;
    size_t total;
};

bool cfg_valid(const coli_moe_config *c, std::string *why) {
    auto bad = [&](const char *m) {
        if (why) *why = m;
        return false;
    };
    if (!c) return bad("cfg is NULL");
    if (c->wfmt != 8 && c->wfmt != 4 && c->wfmt != 2) return bad("wfmt must be 8, 4 or 2");
    const int q = c->wfmt == 2 ? 64 : 32;
    if (c->hidden <= 0 || c->hidden % q || c->hidden > 16384)
        return bad("hidden must be a positive multiple of 32 (64 for int2), <= 16384");
    if (c->inter <= 0 || c->inter % q || c->inter > 16384)
        return bad("inter must be a positive multiple of 32 (64 for int2), <= 16384");
    if (c->n_routed < 0 || c->n_routed > 1024) return bad("n_routed must be in [0, 1024]");
    if (c->n_shared < 0 || c->n_shared > 4) return bad("n_shared must be in [0, 4]");
    if (c->n_routed == 0) {  // a dense layer: no router, shared experts only
        if (c->top_k != 0 || c->n_shared < 1)
            return bad("a layer without routed experts needs top_k = 0 and n_shared >= 1");
        if (!(c->routed_scaling_factor == c->routed_scaling_factor)) return bad("routed_scaling_factor is NaN");
        if (c->max_tokens < 1 || c->max_tokens > (1 << 20)) return bad("max_tokens must be in [1, 2^20]");
        return true;
    }
    if (c->n_group < 1 || c->n_routed % c->n_group) return bad("n_group must divide n_routed");
    if (c->topk_group < 1 || c->topk_group > c->n_group) return bad("topk_group must be in [1, n_group]");
    const int cand = c->topk_group * (c->n_routed / c->n_group);
    if (c->top_k < 1 || c->top_k > 32 || c->top_k > cand)
        return bad("top_k must be in [1, min(32, topk_group * n_routed / n_group)]");
    if (!(c->routed_scaling_factor == c->routed_scaling_factor)) return bad("routed_scaling_factor is NaN");
    if (!(c->expert_top_p == c->expert_top_p)) return bad("expert_top_p is NaN");
    if (c->max_tokens < 1 || c->max_tokens > (1 << 20)) return bad("max_tokens must be in [1, 2^20]");
    return true;
}

WsOffsets layout_of(const coli_moe_config &c) {
    Layout L;
    WsOffsets o{};
    const size_t T = c.max_tokens, E = c.n_routed, S = c.n_shared, k = c.top_k;
    const size_t H = c.hidden, I = c.inter;
    const size_t P = T * (k + S);
    const size_t wstride = (T + 31) / 32;
    o.s = L.add(T * E * 8);
    o.c = L.add(T * E * 8);
    o.idx = L.add(T * k * 4);
    o.w = L.add(T * k * 4);
    o.bitmap = L.add(E * wstride * 4);
    o.prefix = L.add(E * wstride * 4);
    o.counter = L.add(4);
    o.n_active = L.add(4);
    o.active = L.add((E + S) * 4);
    o.off = L.add((E + S + 1) * 4);
    o.act_of = L.add((E + S) * 4);
    o.pair_tok = L.add(P * 4);
    o.pair_slot = L.add(P * 4);
    o.tok_pair = L.add(P * 4);
    o.xq = L.add(T * H);
    o.xd = L.add(T * (H / 32) * 4);
    o.hq = L.add(P * I);
    o.hd = L.add(P * (I / 32) * 4);
    o.e_pairs = (T > (size_t)SMALL_T) ? L.add(P * H * 4) : 0;
    // pair-ordered x codes and scales, and the tensor maps, for the grouped
    // tensor-core path
    o.xg = (T > (size_t)SMALL_T) ? L.add(P * H) : 0;
    o.xdg = (T > (size_t)SMALL_T) ? L.add(P * (H / 32) * 4) : 0;
    o.maps = (T > (size_t)SMALL_T) ? L.add((TC_MAP_W + 3 * (E + S)) * sizeof(CUtensorMap)) : 0;
    o.corr_x = (T > (size_t)SMALL_T) ? L.add(P * 8) : 0;
    o.corr_h = (T > (size_t)SMALL_T) ? L.add(P * 8) : 0;
    o.x_in = L.add(T * H * 4);
    o.y_out = L.add(T * H * 4);
    o.experts = L.add((E + S) * sizeof(ExpertDev));
    o.xrec = L.add(T * (size_t)rec_bytes((int)H));
    o.hrec = L.add(P * (size_t)rec_bytes((int)I));
    o.err = L.add(4);
    o.gbar = L.add(8);
    o.hcnt = L.add((E + S) * 4);
    o.wait_limit = L.add(8);
    o.total = L.total;
    return o;
}

// --- launch helpers --------------------------------------------------------
cudaEvent_t pool_event(coli_moe *m) {
    if (!m->event_pool.empty()) {
        cudaEvent_t e = m->event_pool.back();
        m->event_pool.pop_back();
        return e;
    }
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

struct Launch {
    coli_moe *m;
    cudaStream_t s;
    const char *name;
    cudaEvent_t a = nullptr;
    Launch(coli_moe *m_, cudaStream_t s_, const char *n) : m(m_), s(s_), name(n) {
        if (m && m->profiling) {
            a = pool_event(m);
            if (a) cudaEventRecord(a, s);
        }
    }
    coli_status done() {
        cudaError_t e = cudaGetLastError();
        g_launches.fetch_add(1, std::memory_order_relaxed);
        if (m && m->profiling && a) {
            cudaEvent_t b = pool_event(m);
            if (b) {
                cudaEventRecord(b, s);
                m->pending.push_back({name, a, b});
            }
        }
        if (e != cudaSuccess) return cuda_fail(e, name);
        return COLI_OK;
    }
};

// Set the kernel's shared-memory limit and return its CTAs per SM, once per
// (handle, kernel); later calls (e.g. during CUDA graph capture) only read the cache.
template <typename K>
coli_status prepare(coli_moe *m, K kernel, int threads, size_t smem, int *occ);

template <typename K>
coli_status allow_smem(K kernel, size_t bytes) {
    if (bytes > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)bytes);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    }
    return COLI_OK;
}

template <typename K>
int occupancy(K kernel, int threads, size_t smem) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess)
        return 1;
    return n > 0 ? n : 1;
}

template <typename K>
coli_status prepare(coli_moe *m, K kernel, int threads, size_t smem, int *occ) {
    // the key includes the shared-memory size: the few-token down kernel's
    // footprint depends on T
    const void *key = (const void *)((uintptr_t)(const void *)kernel ^ ((uintptr_t)smem << 40));
    auto it = m->occ_cache.find(key);
    if (it != m->occ_cache.end()) {
        *occ = it->second;
        return COLI_OK;
    }
    coli_status st = allow_smem(kernel, smem);
    if (st != COLI_OK) return st;
    const int o = occupancy(kernel, threads, smem);
    m->occ_cache[key] = o;
    *occ = o;
    return COLI_OK;
}

// --- kernel dispatch by (BITS, VPL) ------------------------------------------
template <int BITS, int VPL>
coli_status launch_gateup_t(coli_moe *m, int max_items, cudaStream_t s) {
    const auto &c = m->cfg;
    auto kern = k_gateup<BITS, VPL>;
    size_t smem = stage_bytes(GROUP_NT, c.hidden) + 2 * ROWS_PER_ITEM * GROUP_NT * 4;
    int occ = 1;
    coli_status st = prepare(m, kern, 256, smem, &occ);
    if (st != COLI_OK) return st;
    int grid = std::min(max_items, m->nsm * occ);
    grid = std::max(grid, 1);
    Launch L(m, s, "gateup_swiglu_q8");
    kern<<<grid, 256, smem, s>>>(m->rw, m->experts_dev, m->xq, m->xd, c.hidden, c.inter, m->hq,
                                 m->hd);
    return L.done();
}

template <int BITS>
coli_status launch_gateup(coli_moe *m, int max_items, cudaStream_t s) {
    switch (pick_vpl(m->cfg.hidden * BITS / 128)) {
        case 1: return launch_gateup_t<BITS, 1>(m, max_items, s);
        case 2: return launch_gateup_t<BITS, 2>(m, max_items, s);
        case 4: return launch_gateup_t<BITS, 4>(m, max_items, s);
        case 6: return launch_gateup_t<BITS, 6>(m, max_items, s);
        case 12: return launch_gateup_t<BITS, 12>(m, max_items, s);
        default: return launch_gateup_t<BITS, 0>(m, max_items, s);
    }
}

template <int BITS, int VPL>
coli_status launch_down_small_t(coli_moe *m, int T, float *out, cudaStream_t s) {
    const auto &c = m->cfg;
    auto kern = k_down_combine<BITS, VPL>;
    const size_t P = (size_t)T * (c.top_k + c.n_shared);
    size_t smem = stage_bytes((int)P, c.inter) + (size_t)GROUP_WARPS * P * DOWN_ROWS * 8;
    int occ = 1;
    coli_status st = prepare(m, kern, 256, smem, &occ);
    if (st != COLI_OK) return st;
    const int groups = c.hidden / DOWN_ROWS;
    int grid = std::min((groups + GROUP_WARPS - 1) / GROUP_WARPS, m->nsm * occ);
    grid = std::max(grid, 1);
    Launch L(m, s, "down_combine");
    kern<<<grid, 256, smem, s>>>(m->rw, m->experts_dev, m->hq, m->hd, T, c.hidden, c.inter,
                                 c.top_k, c.n_shared, out, m->out_partial);
    return L.done();
}

template <int BITS>
coli_status launch_down_small(coli_moe *m, int T, float *out, cudaStream_t s) {
    switch (pick_vpl(m->cfg.inter * BITS / 128)) {
        case 1: return launch_down_small_t<BITS, 1>(m, T, out, s);
        case 2: return launch_down_small_t<BITS, 2>(m, T, out, s);
        case 4: return launch_down_small_t<BITS, 4>(m, T, out, s);
        case 6: return launch_down_small_t<BITS, 6>(m, T, out, s);
        case 12: return launch_down_small_t<BITS, 12>(m, T, out, s);
        default: return launch_down_small_t<BITS, 0>(m, T, out, s);
    }
}

template <int BITS, int VPL>
coli_status launch_down_grouped_t(coli_moe *m, int max_items, cudaStream_t s) {
    const auto &c = m->cfg;
    auto kern = k_down_grouped<BITS, VPL>;
    size_t smem = stage_bytes(GROUP_NT, c.inter);
    int occ = 1;
    coli_status st = prepare(m, kern, 256, smem, &occ);
    if (st != COLI_OK) return st;
    int grid = std::max(1, std::min(max_items, m->nsm * occ));
    Launch L(m, s, "down_grouped");
    kern<<<grid, 256, smem, s>>>(m->rw, m->experts_dev, m->hq, m->hd, c.hidden, c.inter,
                                 m->e_pairs);
    return L.done();
}

template <int BITS>
coli_status launch_down_grouped(coli_moe *m, int max_items, cudaStream_t s) {
    switch (pick_vpl(m->cfg.inter * BITS / 128)) {
        case 1: return launch_down_grouped_t<BITS, 1>(m, max_items, s);
        case 2: return launch_down_grouped_t<BITS, 2>(m, max_items, s);
        case 4: return launch_down_grouped_t<BITS, 4>(m, max_items, s);
        case 6: return launch_down_grouped_t<BITS, 6>(m, max_items, s);
        case 12: return launch_down_grouped_t<BITS, 12>(m, max_items, s);
        default: return launch_down_grouped_t<BITS, 0>(m, max_items, s);
    }
}

size_t select_smem(const coli_moe_config &c) { return select_smem_bytes(c.n_routed, c.n_group); }

// Launch with programmatic stream serialization (PDL) when `pdl` is set: the
// kernel may start while the previous kernel on the stream is finishing and
// waits for it with griddepcontrol.wait before reading its results.
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t s, bool pdl, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Cooperative launch: every CTA of the grid is resident at once (required by
// the front kernel's grid barrier); the launch fails instead of running a
// grid that does not fit.
template <typename... KArgs, typename... Args>
cudaError_t launch_coop(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                        cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ---- few-token path sizing ------------------------------------------------
constexpr int SMEM_BUDGET = 227 * 1024;

struct PipePlan {
    int ns = 0;            // ring stages
    size_t stage = 0;      // bytes per stage
    size_t smem = 0;       // dynamic shared memory
    int stage_rows = 0;    // down: rows per stage
    int grid = 0;
    int rows_cap = 0;      // down: rows per CTA (max)
    int amax = 0, pmax = 0;
    int nh = 0, h_alias = 0, ptr_smem = 0;  // decode kernel: h slots, their placement, pointer table
    int down_span = 1;                       // ring slots per down stage
};

int ring_stages(size_t fixed, size_t stage) {
    if (fixed >= (size_t)SMEM_BUDGET) return 0;
    return (int)std::min<size_t>((SMEM_BUDGET - fixed) / stage, PIPE_MAX_STAGES);
}

PipePlan plan_decode(const coli_moe *m, int T) {
    const auto &c = m->cfg;
    PipePlan p;
    const GuGeom g = gu_geometry(c.hidden, c.wfmt);
    p.grid = m->nsm;  // one CTA per SM, all co-resident
    p.pmax = T * (c.top_k + c.n_shared);
    p.rows_cap = (c.hidden + p.grid - 1) / p.grid;
    const int RBI = c.inter * c.wfmt / 8;
    p.amax = std::min(c.n_routed, T * c.top_k) + c.n_shared;
    auto fixed = [&](int nh, int alias, int ptrs) {
        return decode_smem(T, c.hidden, c.inter, c.n_routed, c.n_shared, c.n_group, c.top_k,
                           p.pmax, g.slices, p.rows_cap, 0, nh, alias, ptrs).total;
    };
    // h slots of their own (filled as soon as each expert's h is complete) as
    // many as fit beside a ring of at least 4 stages; else two slots in the
    // x records' space (filled after the gate/up items)
    p.ptr_smem = c.n_routed + c.n_shared <= DECODE_PTR_SMEM_MAX ? 1 : 0;
    p.nh = 2;
    p.h_alias = 1;
    for (int nh = std::min(p.amax, DECODE_MAX_HSLOTS); nh >= 2; --nh) {
        if (ring_stages(fixed(nh, 0, p.ptr_smem), PIPE_STAGE_MAX) >= 4) {
            p.nh = nh;
            p.h_alias = 0;
            break;
        }
    }
    if (p.h_alias && ring_stages(fixed(2, 1, p.ptr_smem), PIPE_STAGE_MAX) < 3) p.ptr_smem = 0;
    const size_t f = fixed(p.nh, p.h_alias, p.ptr_smem);
    p.ns = ring_stages(f, PIPE_STAGE_MAX);
    // Down stages: a CTA's rows of one expert are fetched in as few bulk
    // copies as possible -- DRAM serves one copy per slice far better than
    // the slice split over several stages -- so with an even ring a down
    // stage takes two adjacent slots.  At most 8 rows per consumer warp.
    p.down_span = p.ns >= 4 ? 2 : 1;
    if (p.down_span == 2) p.ns &= ~1;
    const int cap_rows = p.down_span * PIPE_STAGE_MAX / RBI;
    const int want = (p.rows_cap + PIPE_CONSUMERS - 1) / PIPE_CONSUMERS * PIPE_CONSUMERS;
    int rows = std::min(want, cap_rows >= PIPE_CONSUMERS ? cap_rows / PIPE_CONSUMERS * PIPE_CONSUMERS
                                                         : cap_rows);
    p.stage_rows = std::max(1, std::min(rows, 8 * PIPE_CONSUMERS));
    p.smem = f + (size_t)p.ns * PIPE_STAGE_MAX;
    return p;
}

bool small_path_ok(const coli_moe *m, int T) {
    if (T > PIPE_MAX_TOK || m->cfg.hidden < m->nsm) return false;
    return plan_decode(m, T).ns >= 3;
}

coli_status launch_route(coli_moe *m, const float *x, int T, int32_t *idx, float *w,
                         int do_union, cudaStream_t s) {
    const auto &c = m->cfg;
    const int E = c.n_routed, H = c.hidden;
    if (T <= 8 && !do_union) {
        const size_t smem = select_smem(c) + 4 * (size_t)c.n_routed + 4 * (size_t)T * c.top_k;
        int occ = 1;
        void (*kern)(const float *, int, int, const float *, const float *, int, int, int, int,
                     int, float, RouteWs, uint8_t *, int8_t *, float *, int, int32_t *, float *, float);
        if (T <= 1) kern = k_router_small<1, 4>;
        else if (T <= 2) kern = k_router_small<2, 4>;
        else if (T <= 4) kern = k_router_small<4, 4>;
        else kern = k_router_small<8, 4>;
        coli_status st = prepare(m, kern, 256, smem, &occ);
        if (st != COLI_OK) return st;
        Launch L(m, s, "router");
        kern<<<E, 256, smem, s>>>(x, T, H, m->router_w, m->bias, E, c.n_shared, c.n_group,
                                  c.topk_group, c.top_k, c.routed_scaling_factor, m->rw, nullptr,
                                  nullptr, nullptr, 0, idx, w, c.expert_top_p);
        return L.done();
    }
    if (E > 0) {
        Launch L(m, s, "router_logits");
        if (T <= 8) {
            const int grid = (E + 7) / 8;
            switch (T) {
                case 1: k_route_logits_small<1><<<grid, 256, 0, s>>>(x, T, H, m->router_w, m->bias, E, m->rw.s, m->rw.c); break;
                case 2: k_route_logits_small<2><<<grid, 256, 0, s>>>(x, T, H, m->router_w, m->bias, E, m->rw.s, m->rw.c); break;
                case 3:
                case 4: k_route_logits_small<4><<<grid, 256, 0, s>>>(x, T, H, m->router_w, m->bias, E, m->rw.s, m->rw.c); break;
                default: k_route_logits_small<8><<<grid, 256, 0, s>>>(x, T, H, m->router_w, m->bias, E, m->rw.s, m->rw.c); break;
            }
        } else {
            dim3 grid((T + 63) / 64, (E + 63) / 64);
            k_route_logits_tiled<<<grid, 256, 0, s>>>(x, T, H, m->router_w, m->bias, E, m->rw.s,
                                                      m->rw.c);
        }
        coli_status st = L.done();
        if (st != COLI_OK) return st;
    }
    {
        size_t smem = select_smem(c);
        int occ = 1;
        coli_status st = m ? prepare(m, k_route_select, 256, smem, &occ)
                           : allow_smem(k_route_select, smem);
        if (st != COLI_OK) return st;
        Launch L(m, s, "router_select");
        k_route_select<<<T, 256, smem, s>>>(m->rw, T, E, c.n_shared, c.n_group, c.topk_group,
                                            c.top_k, c.routed_scaling_factor, idx, w, do_union,
                                            c.expert_top_p);
        return L.done();
    }
}

template <int BITS>
coli_status launch_small_path(coli_moe *m, const float *x, int T, float *out, cudaStream_t s) {
    const auto &c = m->cfg;
    const PipePlan p = plan_decode(m, T);
    auto kern = T == 1 ? k_moe_decode<BITS, 1> : k_moe_decode<BITS, PIPE_MAX_TOK>;
    int occ = 1;
    coli_status st = prepare(m, kern, DECODE_THREADS, p.smem, &occ);
    if (st != COLI_OK) return st;
    if (occ < 1) return fail(COLI_EUNSUPPORTED, "decode kernel does not fit on an SM");
    DecodeArgs fa{};
    fa.x = x;
    fa.Wr = m->router_w;
    fa.bias = m->bias;
    fa.T = T;
    fa.H = c.hidden;
    fa.I = c.inter;
    fa.E = c.n_routed;
    fa.S = c.n_shared;
    fa.G = c.n_group;
    fa.gk = c.topk_group;
    fa.k = c.top_k;
    fa.rsf = c.routed_scaling_factor;
    fa.top_p = c.expert_top_p;
    fa.ws = m->rw;
    fa.experts = m->experts_dev;
    fa.xrec = m->xrec;
    fa.xq = m->xq;
    fa.xd = m->xd;
    fa.hrec = m->hrec;
    fa.hq = m->hq;
    fa.hd = m->hd;
    fa.out = out;
    fa.out_partial = m->out_partial;
    fa.err = m->err;
    fa.wait_limit = m->wait_limit;
    fa.gbar = m->gbar;
    fa.hcnt = m->hcnt;
    fa.ns = p.ns;
    fa.pmax = p.pmax;
    fa.rows_cap = p.rows_cap;
    fa.down_rows = p.stage_rows;
    fa.down_span = p.down_span;
    fa.nh = p.nh;
    fa.h_alias = p.h_alias;
    fa.ptr_smem = p.ptr_smem;
    Launch L(m, s, "moe_decode");
    cudaError_t e = launch_coop(kern, dim3(p.grid), dim3(DECODE_THREADS), p.smem, s, fa);
    if (e != cudaSuccess) return cuda_fail(e, "moe_decode launch");
    return L.done();
}

coli_status quant_q8_launch(coli_moe *m, const float *x, int64_t rows, int64_t len, int8_t *q,
                            float *d, cudaStream_t s) {
    const int64_t nblocks = rows * (len / COLI_QBLK);
    if (nblocks == 0) return COLI_OK;
    const int64_t warps = 8;
    int64_t grid = std::min<int64_t>((nblocks + warps - 1) / warps, (int64_t)sm_count() * 16);
    Launch L(m, s, "quant_q8");
    k_quant_q8<<<(unsigned)grid, 256, 0, s>>>(x, nblocks, q, d);
    return L.done();
}

coli_status check_handle(coli_moe *m) {
    if (!m) return fail(COLI_EINVAL, "handle is NULL");
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != m->device)
        return fail(COLI_EINVAL, "current device %d is not the handle's device %d", dev, m->device);
    return COLI_OK;
}

// 2-D tensor maps through the driver's encoder, fetched from the runtime (no
// link against the driver library).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)p;
    });
    return fn;
}

// rows x cols matrix (cols contiguous, row pitch in bytes), box box_rows x box_cols
bool encode_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t rows, uint64_t cols,
               uint64_t pitch, uint32_t box_rows, uint32_t box_cols) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (!fn || !base) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {pitch};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor-core grouped GEMMs for many tokens: both reductions in whole
// stages of 8 blocks and both row counts in whole tiles.
bool tc_path_ok(const coli_moe *m) {
    const auto &c = m->cfg;
    return m->e_pairs && m->tc_maps && c.hidden % (TC_BPS * 32) == 0 && c.inter % (TC_BPS * 32) == 0 &&
           c.inter % TC_M == 0 && c.hidden % (2 * TC_M) == 0;
}

template <int BITS>
coli_status launch_grouped_tc(coli_moe *m, int T, int down, cudaStream_t s) {
    const auto &c = m->cfg;
    const int max_active = std::min(c.n_routed, T * c.top_k) + c.n_shared;
    const size_t smem = tc_layout(BITS, max_active).total;
    auto kern = k_grouped_tc<BITS>;
    int occ = 1;
    coli_status st = prepare(m, kern, TC_THREADS, smem, &occ);
    if (st != COLI_OK) return st;
    if (occ < 1) return fail(COLI_EUNSUPPORTED, "grouped tensor-core kernel does not fit on an SM");
    TcArgs ta{};
    ta.ws = m->rw;
    ta.experts = m->experts_dev;
    ta.down = down;
    ta.K = down ? c.inter : c.hidden;
    ta.I = c.inter;
    ta.H = c.hidden;
    ta.maps = m->maps_dev;
    ta.map_b = down ? TC_MAP_HQ : TC_MAP_XG;
    ta.map_d = down ? TC_MAP_HD : TC_MAP_XD;
    ta.corr = down ? m->corr_h : m->corr_x;
    ta.hq = m->hq;
    ta.hd = m->hd;
    ta.e_pairs = m->e_pairs;
    ta.err = m->err;
    ta.wait_limit = m->wait_limit;
    Launch L(m, s, down ? "down_tc" : "gateup_tc");
    kern<<<m->nsm, TC_THREADS, smem, s>>>(ta);
    return L.done();
}

template <int BITS>
coli_status launch_tc_path(coli_moe *m, int T, float *out, cudaStream_t s) {
    const auto &c = m->cfg;
    const double off = BITS == 4 ? 8.0 : 2.0;  // unsigned weight operands: code + off
    {
        Launch L(m, s, "gather_pairs");
        k_gather_pairs<<<m->nsm * 8, 256, 0, s>>>(m->rw, m->xq, m->xd, c.hidden, m->xg, m->xdg);
        coli_status st = L.done();
        if (st != COLI_OK) return st;
    }
    if (BITS != 8) {
        Launch L(m, s, "pair_offsets");
        k_pair_offsets<<<m->nsm * 8, 256, 0, s>>>(m->rw, m->xg, m->xdg, c.hidden, off, m->corr_x);
        coli_status st = L.done();
        if (st != COLI_OK) return st;
    }
    coli_status st = launch_grouped_tc<BITS>(m, T, 0, s);
    if (st != COLI_OK) return st;
    if (BITS != 8) {
        Launch L(m, s, "pair_offsets");
        k_pair_offsets<<<m->nsm * 8, 256, 0, s>>>(m->rw, m->hq, m->hd, c.inter, off, m->corr_h);
        st = L.done();
        if (st != COLI_OK) return st;
    }
    st = launch_grouped_tc<BITS>(m, T, 1, s);
    if (st != COLI_OK) return st;
    Launch L(m, s, "combine");
    const int64_t n = (int64_t)T * c.hidden;
    int grid = (int)std::min<int64_t>((n + 255) / 256, (int64_t)m->nsm * 8);
    k_combine<<<grid, 256, 0, s>>>(m->rw, m->e_pairs, T, c.hidden, c.top_k, c.n_shared, out,
                                   m->out_partial);
    return L.done();
}

coli_status forward_impl(coli_moe *m, const float *x, int T, float *out, cudaStream_t s) {
    const auto &c = m->cfg;
    coli_status st;
    if (small_path_ok(m, T)) {
        switch (c.wfmt) {
            case 8: st = launch_small_path<8>(m, x, T, out, s); break;
            case 4: st = launch_small_path<4>(m, x, T, out, s); break;
            default: st = launch_small_path<2>(m, x, T, out, s); break;
        }
        if (st == COLI_OK) m->last_T = T;
        return st;
    }
    st = quant_q8_launch(m, x, T, c.hidden, m->xq, m->xd, s);
    if (st != COLI_OK) return st;
    st = launch_route(m, x, T, m->rw.idx, m->rw.w, 1, s);
    if (st != COLI_OK) return st;
    if (tc_path_ok(m) && !m->no_tc) {
        switch (c.wfmt) {
            case 8: st = launch_tc_path<8>(m, T, out, s); break;
            case 4: st = launch_tc_path<4>(m, T, out, s); break;
            default: st = launch_tc_path<2>(m, T, out, s); break;
        }
        if (st == COLI_OK) m->last_T = T;
        return st;
    }
    const int max_active = std::min(c.n_routed, T * c.top_k) + c.n_shared;
    const int gu_items = max_active * (c.inter / ROWS_PER_ITEM);
    switch (c.wfmt) {
        case 8: st = launch_gateup<8>(m, gu_items, s); break;
        case 4: st = launch_gateup<4>(m, gu_items, s); break;
        default: st = launch_gateup<2>(m, gu_items, s); break;
    }
    if (st != COLI_OK) return st;
    const size_t P = (size_t)T * (c.top_k + c.n_shared);
    const size_t small_smem = stage_bytes((int)P, c.inter) + (size_t)GROUP_WARPS * P * DOWN_ROWS * 8;
    if (T <= SMALL_T && small_smem <= (size_t)MAX_SMEM) {
        switch (c.wfmt) {
            case 8: st = launch_down_small<8>(m, T, out, s); break;
            case 4: st = launch_down_small<4>(m, T, out, s); break;
            default: st = launch_down_small<2>(m, T, out, s); break;
        }
        if (st != COLI_OK) return st;
    } else {
        if (!m->e_pairs) return fail(COLI_EUNSUPPORTED, "T=%d needs the grouped down path", T);
        const int dn_items = max_active * (c.hidden / ROWS_PER_ITEM);
        switch (c.wfmt) {
            case 8: st = launch_down_grouped<8>(m, dn_items, s); break;
            case 4: st = launch_down_grouped<4>(m, dn_items, s); break;
            default: st = launch_down_grouped<2>(m, dn_items, s); break;
        }
        if (st != COLI_OK) return st;
        Launch L(m, s, "combine");
        const int64_t n = (int64_t)T * c.hidden;
        int grid = (int)std::min<int64_t>((n + 255) / 256, (int64_t)m->nsm * 8);
        k_combine<<<grid, 256, 0, s>>>(m->rw, m->e_pairs, T, c.hidden, c.top_k, c.n_shared, out,
                                   m->out_partial);
        st = L.done();
        if (st != COLI_OK) return st;
    }
    m->last_T = T;
    return COLI_OK;
}

__global__ void k_dbg_wait_probe(int *err) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, err);  // nothing arrives: gives up
}

__global__ void k_gather_h(const int32_t *__restrict__ tok_pair, const int8_t *__restrict__ hq,
                           const float *__restrict__ hd, int T, int slots, int I,
                           int8_t *__restrict__ hq_out, float *__restrict__ hd_out) {
    const int ts = blockIdx.x;  // (token, slot)
    if (ts >= T * slots) return;
    const int p = tok_pair[ts];  // -1: an expert another handle computes (zeros here)
    for (int i = threadIdx.x; i < I; i += blockDim.x) {
        if (hq_out) hq_out[(int64_t)ts * I + i] = p < 0 ? (int8_t)0 : hq[(int64_t)p * I + i];
        if (hd_out && i < I / COLI_QBLK)
            hd_out[(int64_t)ts * (I / COLI_QBLK) + i] = p < 0 ? 0.0f : hd[(int64_t)p * (I / COLI_QBLK) + i];
    }
}

// Sum of the partial outputs of expert-parallel handles, in part order:
// out[i] = fp32( parts[0][i] + parts[1][i] + ... ), fp64 throughout.
__global__ void k_sum_partials(const double *__restrict__ parts, int n_parts, int64_t n,
                               float *__restrict__ out) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        double acc = 0.0;
        for (int r = 0; r < n_parts; ++r) acc += parts[(int64_t)r * n + i];
        out[i] = (float)acc;
    }
}

// ---------------------------------------------------------------------------
// Scratch of coli_router_static: fp64 sigmoid scores s [T][E] and choice
// scores c [T][E] for at most ROUTER_STATIC_MAX_T tokens and
// ROUTER_STATIC_MAX_E experts, then the last-CTA ticket.  A file-scope device
// array: every GPU that loads the library holds it until the process exits,
// and every coli_router_static call on that GPU shares it.
constexpr int ROUTER_STATIC_MAX_T = 8;
constexpr int ROUTER_STATIC_MAX_E = 1024;
constexpr size_t ROUTER_STATIC_SC_BYTES = (size_t)ROUTER_STATIC_MAX_T * ROUTER_STATIC_MAX_E * 8;
constexpr size_t ROUTER_STATIC_BYTES = 2 * ROUTER_STATIC_SC_BYTES + 256;
static __device__ __align__(256) unsigned char g_router_scratch[ROUTER_STATIC_BYTES];

// Device address of g_router_scratch per device, looked up once per device
// with that device current.  In host code the symbol is only a stand-in.
std::mutex g_router_scratch_mu;
void *g_router_scratch_dev[128] = {nullptr};

coli_status router_scratch_address(int dev, void **out) {
    if (dev < 0 || dev >= 128) return fail(COLI_EUNSUPPORTED, "device ordinal %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_router_scratch_mu);
    if (!g_router_scratch_dev[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_router_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(router scratch)");
        g_router_scratch_dev[dev] = p;
    }
    *out = g_router_scratch_dev[dev];
    return COLI_OK;
}

}  // namespace

// ===========================================================================
extern "C" {

const char *coli_status_str(coli_status s) {
    switch (s) {
        case COLI_OK: return "COLI_OK";
        case COLI_EINVAL: return "COLI_EINVAL";
        case COLI_ENOMEM: return "COLI_ENOMEM";
        case COLI_ECUDA: return "COLI_ECUDA";
        case COLI_EUNSUPPORTED: return "COLI_EUNSUPPORTED";
        case COLI_ETIMEOUT: return "COLI_ETIMEOUT";
    }
    return "COLI_UNKNOWN";
}

const char *coli_last_error(void) { return g_last_error.c_str(); }
int coli_abi_version(void) { return COLI_ABI_VERSION; }
uint64_t coli_launch_count(void) { return g_launches.load(); }

coli_status coli_quant_q8(const float *x, int64_t rows, int64_t len, int8_t *q, float *d,
                          coli_stream_t stream) {
    g_last_error.clear();
    if (rows < 0 || len <= 0 || len % COLI_QBLK) return fail(COLI_EINVAL, "len must be a positive multiple of 32, rows >= 0");
    if (rows == 0) return COLI_OK;
    if (!x || !q || !d) return fail(COLI_EINVAL, "null pointer");
    if (!aligned16(x) || !aligned16(q) || !aligned16(d)) return fail(COLI_EINVAL, "pointers must be 16-byte aligned");
    return quant_q8_launch(nullptr, x, rows, len, q, d, (cudaStream_t)stream);
}

coli_status coli_quant_weights(const float *w, int64_t rows, int64_t K, int wfmt, void *codes,
                               float *scales, coli_stream_t stream) {
    g_last_error.clear();
    if (wfmt != 8 && wfmt != 4 && wfmt != 2) return fail(COLI_EINVAL, "wfmt must be 8, 4 or 2");
    if (rows < 0 || K <= 0 || K % (wfmt == 2 ? 64 : 32))
        return fail(COLI_EINVAL, "K must be a positive multiple of 32 (64 for int2)");
    if (rows == 0) return COLI_OK;
    if (!w || !codes || !scales) return fail(COLI_EINVAL, "null pointer");
    if (!aligned16(w) || !aligned16(codes) || !aligned16(scales)) return fail(COLI_EINVAL, "pointers must be 16-byte aligned");
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t grid = std::min<int64_t>((rows + 7) / 8, (int64_t)sm_count() * 16);
    Launch L(nullptr, s, "quant_weights");
    switch (wfmt) {
        case 8: k_quant_weights<8><<<(unsigned)grid, 256, 0, s>>>(w, rows, K, (uint32_t *)codes, scales); break;
        case 4: k_quant_weights<4><<<(unsigned)grid, 256, 0, s>>>(w, rows, K, (uint32_t *)codes, scales); break;
        default: k_quant_weights<2><<<(unsigned)grid, 256, 0, s>>>(w, rows, K, (uint32_t *)codes, scales); break;
    }
    return L.done();
}

coli_status coli_requant_fp8(const void *w_fp8, const float *block_scale, int64_t rows, int64_t K,
                            int64_t block, int wfmt, void *codes, float *scales,
                            coli_stream_t stream) {
    g_last_error.clear();
    if (wfmt != 8 && wfmt != 4 && wfmt != 2) return fail(COLI_EINVAL, "wfmt must be 8, 4 or 2");
    if (rows < 0 || K <= 0 || K % (wfmt == 2 ? 64 : 32))
        return fail(COLI_EINVAL, "K must be a positive multiple of 32 (64 for int2)");
    if (block <= 0 || block % 16) return fail(COLI_EINVAL, "block must be a positive multiple of 16");
    if (rows == 0) return COLI_OK;
    if (!w_fp8 || !block_scale || !codes || !scales) return fail(COLI_EINVAL, "null pointer");
    if (!aligned16(w_fp8) || !aligned16(codes) || !((uintptr_t)block_scale % 4 == 0) ||
        !((uintptr_t)scales % 4 == 0))
        return fail(COLI_EINVAL, "w_fp8 and codes must be 16-byte aligned, scales 4-byte aligned");
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t grid = std::min<int64_t>((rows + 7) / 8, (int64_t)sm_count() * 16);
    const uint8_t *w8 = (const uint8_t *)w_fp8;
    uint8_t *c = (uint8_t *)codes;
    Launch L(nullptr, s, "requant_fp8");
    switch (wfmt) {
        case 8: k_requant_fp8<8><<<(unsigned)grid, 256, 0, s>>>(w8, block_scale, rows, K, block, c, scales); break;
        case 4: k_requant_fp8<4><<<(unsigned)grid, 256, 0, s>>>(w8, block_scale, rows, K, block, c, scales); break;
        default: k_requant_fp8<2><<<(unsigned)grid, 256, 0, s>>>(w8, block_scale, rows, K, block, c, scales); break;
    }
    return L.done();
}

size_t coli_moe_workspace_bytes(const coli_moe_config *cfg) {
    if (!cfg_valid(cfg, nullptr)) return 0;
    return layout_of(*cfg).total;
}

coli_status coli_moe_create(const coli_moe_config *cfg, const float *router_w, const float *bias,
                            const coli_expert *experts, coli_moe **out) {
    g_last_error.clear();
    if (!out) return fail(COLI_EINVAL, "out is NULL");
    *out = nullptr;
    std::string why;
    if (!cfg_valid(cfg, &why)) return fail(COLI_EINVAL, "invalid config: %s", why.c_str());
    if (!experts || (cfg->n_routed > 0 && (!router_w || !bias)))
        return fail(COLI_EINVAL, "null router/bias/experts");
    if (!aligned16(router_w) || !aligned16(bias)) return fail(COLI_EINVAL, "router pointers must be 16-byte aligned");
    const int n = cfg->n_routed + cfg->n_shared;
    std::vector<ExpertDev> host(n);
    for (int e = 0; e < n; ++e) {
        const coli_qmat *mm[3] = {&experts[e].gate, &experts[e].up, &experts[e].down};
        QMatDev *dd[3] = {&host[e].gate, &host[e].up, &host[e].down};
        for (int j = 0; j < 3; ++j) {
            if (!mm[j]->codes || !mm[j]->scales) return fail(COLI_EINVAL, "expert %d matrix %d is NULL", e, j);
            if (!aligned16(mm[j]->codes) || !aligned16(mm[j]->scales))
                return fail(COLI_EINVAL, "expert %d matrix %d is not 16-byte aligned", e, j);
            dd[j]->codes = (const uint8_t *)mm[j]->codes;
            dd[j]->scales = mm[j]->scales;
        }
    }
    coli_moe *m = new (std::nothrow) coli_moe();
    if (!m) return fail(COLI_ENOMEM, "host allocation failed");
    m->cfg = *cfg;
    m->router_w = router_w;
    m->bias = bias;
    cudaGetDevice(&m->device);
    m->nsm = sm_count();
    m->no_tc = getenv("COLI_NO_TC") && strcmp(getenv("COLI_NO_TC"), "1") == 0;
    const WsOffsets o = layout_of(*cfg);
    if (getenv("COLI_FAULT") && strcmp(getenv("COLI_FAULT"), "alloc") == 0) {
        delete m;
        return fail(COLI_ENOMEM, "injected allocation failure (COLI_FAULT=alloc)");
    }
    cudaError_t e = cudaMalloc(&m->ws_base, o.total);
    if (e != cudaSuccess) {
        delete m;
        return cuda_fail(e, "cudaMalloc(workspace)");
    }
    m->ws_bytes = o.total;
    char *b = (char *)m->ws_base;
    m->rw.s = (double *)(b + o.s);
    m->rw.c = (double *)(b + o.c);
    m->rw.idx = (int32_t *)(b + o.idx);
    m->rw.w = (float *)(b + o.w);
    m->rw.bitmap = (uint32_t *)(b + o.bitmap);
    m->rw.prefix = (int32_t *)(b + o.prefix);
    m->rw.counter = (uint32_t *)(b + o.counter);
    m->rw.n_active = (int32_t *)(b + o.n_active);
    m->rw.active = (int32_t *)(b + o.active);
    m->rw.off = (int32_t *)(b + o.off);
    m->rw.act_of = (int32_t *)(b + o.act_of);
    m->rw.pair_tok = (int32_t *)(b + o.pair_tok);
    m->rw.pair_slot = (int32_t *)(b + o.pair_slot);
    m->rw.tok_pair = (int32_t *)(b + o.tok_pair);
    m->rw.wstride = (cfg->max_tokens + 31) / 32;
    m->rw.e_lo = 0;  // every routed and shared expert, until coli_moe_set_experts
    m->rw.e_hi = cfg->n_routed;
    m->rw.own_shared = 1;
    m->xq = (int8_t *)(b + o.xq);
    m->xd = (float *)(b + o.xd);
    m->hq = (int8_t *)(b + o.hq);
    m->hd = (float *)(b + o.hd);
    m->e_pairs = o.e_pairs ? (float *)(b + o.e_pairs) : nullptr;
    m->xg = o.xg ? (int8_t *)(b + o.xg) : nullptr;
    m->xdg = o.xdg ? (float *)(b + o.xdg) : nullptr;
    m->maps_dev = o.maps ? (CUtensorMap *)(b + o.maps) : nullptr;
    m->corr_x = o.corr_x ? (double *)(b + o.corr_x) : nullptr;
    m->corr_h = o.corr_h ? (double *)(b + o.corr_h) : nullptr;
    m->x_in = (float *)(b + o.x_in);
    m->y_out = (float *)(b + o.y_out);
    m->experts_dev = (ExpertDev *)(b + o.experts);
    m->xrec = (uint8_t *)(b + o.xrec);
    m->hrec = (uint8_t *)(b + o.hrec);
    m->err = (int *)(b + o.err);
    m->gbar = (unsigned long long *)(b + o.gbar);
    m->hcnt = (int *)(b + o.hcnt);
    m->wait_limit = (long long *)(b + o.wait_limit);
    e = cudaMemset(m->ws_base, 0, o.total);
    if (e == cudaSuccess)
        e = cudaMemcpy(m->experts_dev, host.data(), sizeof(ExpertDev) * n, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) {
        const long long lim = WAIT_LIMIT_CYCLES;
        e = cudaMemcpy(m->wait_limit, &lim, sizeof lim, cudaMemcpyHostToDevice);
    }
    if (e == cudaSuccess && m->maps_dev) {
        // the tensor-core path's maps; any shape or alignment the copy engine
        // refuses leaves that path off (the CUDA-core grouped kernels run)
        const uint64_t H = cfg->hidden, I = cfg->inter, P = (uint64_t)cfg->max_tokens * (cfg->top_k + cfg->n_shared);
        const int bits = cfg->wfmt;
        std::vector<CUtensorMap> maps(TC_MAP_W + 3 * n);
        bool ok = H % (TC_BPS * 32) == 0 && I % (TC_BPS * 32) == 0;
        const uint32_t gb = (uint32_t)tc_group_bytes(bits);
        ok = ok && encode_2d(&maps[TC_MAP_XG], CU_TENSOR_MAP_DATA_TYPE_UINT8, m->xg, P, H, H, TC_N, 32);
        ok = ok && encode_2d(&maps[TC_MAP_XD], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, m->xdg, P, H / 32, H / 8, TC_N, TC_BPS);
        ok = ok && encode_2d(&maps[TC_MAP_HQ], CU_TENSOR_MAP_DATA_TYPE_UINT8, m->hq, P, I, I, TC_N, 32);
        ok = ok && encode_2d(&maps[TC_MAP_HD], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, m->hd, P, I / 32, I / 8, TC_N, TC_BPS);
        for (int i = 0; ok && i < n; ++i) {
            const uint64_t gu_pitch = H * bits / 8, dn_pitch = I * bits / 8;
            ok = encode_2d(&maps[TC_MAP_W + 3 * i], CU_TENSOR_MAP_DATA_TYPE_UINT8, host[i].gate.codes, I, gu_pitch,
                           gu_pitch, TC_M, gb) &&
                 encode_2d(&maps[TC_MAP_W + 3 * i + 1], CU_TENSOR_MAP_DATA_TYPE_UINT8, host[i].up.codes, I,
                           gu_pitch, gu_pitch, TC_M, gb) &&
                 encode_2d(&maps[TC_MAP_W + 3 * i + 2], CU_TENSOR_MAP_DATA_TYPE_UINT8, host[i].down.codes, H,
                           dn_pitch, dn_pitch, TC_M, gb);
        }
        if (ok) {
            e = cudaMemcpy(m->maps_dev, maps.data(), sizeof(CUtensorMap) * maps.size(), cudaMemcpyHostToDevice);
            m->tc_maps = e == cudaSuccess;
        }
    }
    if (e != cudaSuccess) {
        cudaFree(m->ws_base);
        delete m;
        return cuda_fail(e, "workspace init");
    }
    *out = m;
    return COLI_OK;
}

coli_status coli_router(coli_moe *m, const float *x, int T, int32_t *idx, float *w,
                        coli_stream_t stream) {
    g_last_error.clear();
    coli_status st = check_handle(m);
    if (st != COLI_OK) return st;
    if (T < 1 || T > m->cfg.max_tokens) return fail(COLI_EINVAL, "T=%d outside [1, max_tokens=%d]", T, m->cfg.max_tokens);
    if (!x || !idx || !w) return fail(COLI_EINVAL, "null pointer");
    if (!aligned16(x) || !aligned16(idx) || !aligned16(w)) return fail(COLI_EINVAL, "pointers must be 16-byte aligned");
    if (m->cfg.n_routed == 0) return fail(COLI_EINVAL, "a dense layer has no router");
    return launch_route(m, x, T, idx, w, 0, (cudaStream_t)stream);
}

coli_status coli_moe_forward(coli_moe *m, const float *x, int T, float *out, coli_stream_t stream) {
    g_last_error.clear();
    coli_status st = check_handle(m);
    if (st != COLI_OK) return st;
    if (T < 1 || T > m->cfg.max_tokens) return fail(COLI_EINVAL, "T=%d outside [1, max_tokens=%d]", T, m->cfg.max_tokens);
    if (!x || !out) return fail(COLI_EINVAL, "null pointer");
    if (!aligned16(x) || !aligned16(out)) return fail(COLI_EINVAL, "pointers must be 16-byte aligned");
    const size_t bytes = (size_t)T * m->cfg.hidden * 4;
    const char *xa = (const char *)x, *oa = (const char *)out;
    if (xa < oa + bytes && oa < xa + bytes) return fail(COLI_EINVAL, "out must not alias x");
    return forward_impl(m, x, T, out, (cudaStream_t)stream);
}

coli_status coli_moe_set_experts(coli_moe *m, int e_lo, int e_hi, int own_shared) {
    g_last_error.clear();
    coli_status st = check_handle(m);
    if (st != COLI_OK) return st;
    if (e_lo < 0 || e_hi < e_lo || e_hi > m->cfg.n_routed)
        return fail(COLI_EINVAL, "expert range [%d, %d) outside [0, %d]", e_lo, e_hi, m->cfg.n_routed);
    m->rw.e_lo = e_lo;
    m->rw.e_hi = e_hi;
    m->rw.own_shared = own_shared ? 1 : 0;
    return COLI_OK;
}

coli_status coli_moe_forward_partial(coli_moe *m, const float *x, int T, double *y_partial,
                                     coli_stream_t stream) {
    g_last_error.clear();
    coli_status st = check_handle(m);
    if (st != COLI_OK) return st;
    if (T < 1 || T > m->cfg.max_tokens) return fail(COLI_EINVAL, "T=%d outside [1, max_tokens=%d]", T, m->cfg.max_tokens);
    if (!x || !y_partial) return fail(COLI_EINVAL, "null pointer");
    if (!aligned16(x) || !aligned16(y_partial)) return fail(COLI_EINVAL, "pointers must be 16-byte aligned");
    const size_t xb = (size_t)T * m->cfg.hidden * 4, yb = 2 * xb;
    const char *xa = (const char *)x, *ya = (const char *)y_partial;
    if (xa < ya + yb && ya < xa + xb) return fail(COLI_EINVAL, "y_partial must not alias x");
    m->out_partial = y_partial;
    st = forward_impl(m, x, T, nullptr, (cudaStream_t)stream);
    m->out_partial = nullptr;
    return st;
}

coli_status coli_combine_partials(const double *parts, int n_parts, int64_t n, float *out,
                                  coli_stream_t stream) {
    g_last_error.clear();
    if (n_parts < 1 || n < 0) return fail(COLI_EINVAL, "n_parts must be >= 1 and n >= 0");
    if (n == 0) return COLI_OK;
    if (!parts || !out) return fail(COLI_EINVAL, "null pointer");
    if (!aligned16(parts) || !aligned16(out)) return fail(COLI_EINVAL, "pointers must be 16-byte aligned");
    cudaStream_t s = (cudaStream_t)stream;
    const int grid = (int)std::min<int64_t>((n + 255) / 256, (int64_t)sm_count() * 8);
    Launch L(nullptr, s, "sum_partials");
    k_sum_partials<<<grid, 256, 0, s>>>(parts, n_parts, n, out);
    return L.done();
}

coli_status coli_moe_forward_host(coli_moe *m, const float *x_host, int T, float *out_host,
                                  coli_stream_t stream) {
    g_last_error.clear();
    coli_status st = check_handle(m);
    if (st != COLI_OK) return st;
    if (T < 1 || T > m->cfg.max_tokens) return fail(COLI_EINVAL, "T=%d outside [1, max_tokens=%d]", T, m->cfg.max_tokens);
    if (!x_host || !out_host) return fail(COLI_EINVAL, "null pointer");
    cudaStream_t s = (cudaStream_t)stream;
    const size_t bytes = (size_t)T * m->cfg.hidden * 4;
    COLI_CUDA(cudaMemcpyAsync(m->x_in, x_host, bytes, cudaMemcpyHostToDevice, s), "copy x in");
    st = forward_impl(m, m->x_in, T, m->y_out, s);
    if (st != COLI_OK) return st;
    COLI_CUDA(cudaMemcpyAsync(out_host, m->y_out, bytes, cudaMemcpyDeviceToHost, s), "copy out");
    COLI_CUDA(cudaStreamSynchronize(s), "stream synchronize");
    return COLI_OK;
}

void coli_moe_destroy(coli_moe *m) {
    if (!m) return;
    int prev = -1;
    cudaGetDevice(&prev);
    if (prev != m->device) cudaSetDevice(m->device);
    cudaDeviceSynchronize();
    for (auto &p : m->pending) {
        cudaEventDestroy(p.a);
        cudaEventDestroy(p.b);
    }
    for (auto e : m->event_pool) cudaEventDestroy(e);
    cudaFree(m->ws_base);
    if (prev >= 0 && prev != m->device) cudaSetDevice(prev);
    delete m;
}

coli_status coli_moe_profile(coli_moe *m, int enable) {
    g_last_error.clear();
    if (!m) return fail(COLI_EINVAL, "handle is NULL");
    m->profiling = enable != 0;
    return COLI_OK;
}

coli_status coli_moe_profile_read(coli_moe *m, coli_kernel_time *out, int max_entries,
                                  int *n_entries) {
    g_last_error.clear();
    if (!m || !n_entries || (max_entries > 0 && !out)) return fail(COLI_EINVAL, "bad arguments");
    std::vector<std::pair<const char *, std::pair<int, double>>> acc;
    for (auto &p : m->pending) {
        float ms = 0.0f;
        cudaError_t e = cudaEventSynchronize(p.b);
        if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, p.a, p.b);
        if (e != cudaSuccess) return cuda_fail(e, "profile events");
        bool found = false;
        for (auto &a : acc)
            if (strcmp(a.first, p.name) == 0) {
                a.second.first += 1;
                a.second.second += ms;
                found = true;
            }
        if (!found) acc.push_back({p.name, {1, (double)ms}});
        m->event_pool.push_back(p.a);
        m->event_pool.push_back(p.b);
    }
    m->pending.clear();
    int n = 0;
    for (auto &a : acc) {
        if (n < max_entries) out[n] = coli_kernel_time{a.first, a.second.first, a.second.second};
        ++n;
    }
    *n_entries = n;
    return COLI_OK;
}

coli_status coli_moe_device_status(coli_moe *m, coli_stream_t stream) {
    g_last_error.clear();
    coli_status st = check_handle(m);
    if (st != COLI_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    int word = 0;
    COLI_CUDA(cudaMemcpyAsync(&word, m->err, sizeof(int), cudaMemcpyDeviceToHost, s), "read error word");
    COLI_CUDA(cudaStreamSynchronize(s), "stream synchronize");
    if (word != 0) {
        COLI_CUDA(cudaMemsetAsync(m->err, 0, sizeof(int), s), "clear error word");
        COLI_CUDA(cudaStreamSynchronize(s), "stream synchronize");
        return fail(COLI_ETIMEOUT, "a device-side wait gave up (error word %d)", word);
    }
    return COLI_OK;
}

coli_status coli_router_static(const coli_moe_config *cfg, const float *router_w,
                               const float *bias, const float *x, int T, int32_t *idx, float *w,
                               coli_stream_t stream) {
    g_last_error.clear();
    std::string why;
    if (!cfg_valid(cfg, &why)) return fail(COLI_EINVAL, "invalid config: %s", why.c_str());
    if (cfg->n_routed == 0) return fail(COLI_EINVAL, "a dense layer has no router");
    if (T < 1 || T > ROUTER_STATIC_MAX_T)
        return fail(COLI_EINVAL, "coli_router_static takes 1 <= T <= %d tokens (got %d)",
                    ROUTER_STATIC_MAX_T, T);
    if (cfg->n_routed > ROUTER_STATIC_MAX_E)
        return fail(COLI_EINVAL, "coli_router_static takes at most %d routed experts (got %d)",
                    ROUTER_STATIC_MAX_E, cfg->n_routed);
    if (!router_w || !bias || !x || !idx || !w) return fail(COLI_EINVAL, "null pointer");
    if (!aligned16(router_w) || !aligned16(bias) || !aligned16(x) || !aligned16(idx) || !aligned16(w))
        return fail(COLI_EINVAL, "pointers must be 16-byte aligned");
    int dev = 0;
    COLI_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
    void *base = nullptr;
    coli_status st = router_scratch_address(dev, &base);
    if (st != COLI_OK) return st;
    const int E = cfg->n_routed;
    RouteWs rw{};
    rw.s = (double *)base;
    rw.c = (double *)((char *)base + ROUTER_STATIC_SC_BYTES);
    rw.counter = (uint32_t *)((char *)base + 2 * ROUTER_STATIC_SC_BYTES);
    cudaStream_t s = (cudaStream_t)stream;
    // the ticket must start at zero; s and c are fully written before use
    COLI_CUDA(cudaMemsetAsync(rw.counter, 0, sizeof(uint32_t), s), "clear router ticket");
    const size_t smem = select_smem(*cfg) + 4 * (size_t)E + 4 * (size_t)T * cfg->top_k;
    void (*kern)(const float *, int, int, const float *, const float *, int, int, int, int, int,
                 float, RouteWs, uint8_t *, int8_t *, float *, int, int32_t *, float *, float);
    if (T <= 1) kern = k_router_small<1, 4>;
    else if (T <= 2) kern = k_router_small<2, 4>;
    else if (T <= 4) kern = k_router_small<4, 4>;
    else kern = k_router_small<8, 4>;
    st = allow_smem(kern, smem);
    if (st != COLI_OK) return st;
    Launch L(nullptr, s, "router_static");
    kern<<<E, 256, smem, s>>>(x, T, cfg->hidden, router_w, bias, E, cfg->n_shared, cfg->n_group,
                              cfg->topk_group, cfg->top_k, cfg->routed_scaling_factor, rw, nullptr,
                              nullptr, nullptr, 0, idx, w, cfg->expert_top_p);
    return L.done();
}

coli_status coli_dbg_wait_probe(coli_moe *m, coli_stream_t stream) {
    g_last_error.clear();
    coli_status st = check_handle(m);
    if (st != COLI_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    Launch L(nullptr, s, "dbg_wait_probe");
    k_dbg_wait_probe<<<1, 32, 0, s>>>(m->err);
    return L.done();
}

coli_status coli_dbg_set_wait_limit(coli_moe *m, long long cycles, coli_stream_t stream) {
    g_last_error.clear();
    coli_status st = check_handle(m);
    if (st != COLI_OK) return st;
    const long long lim = cycles > 0 && cycles < WAIT_LIMIT_CYCLES ? cycles : WAIT_LIMIT_CYCLES;
    cudaStream_t s = (cudaStream_t)stream;
    // pageable source: the copy has completed when the call returns
    COLI_CUDA(cudaMemcpyAsync(m->wait_limit, &lim, sizeof lim, cudaMemcpyHostToDevice, s),
              "wait limit copy");
    COLI_CUDA(cudaStreamSynchronize(s), "wait limit copy");
    return COLI_OK;
}

coli_status coli_dbg_block_sums(const void *codes, int wfmt, int64_t rows, int64_t K,
                                const int8_t *xq, int T, int32_t *S, coli_stream_t stream) {
    g_last_error.clear();
    if (wfmt != 8 && wfmt != 4 && wfmt != 2) return fail(COLI_EINVAL, "wfmt must be 8, 4 or 2");
    if (rows < 1 || T < 1 || T > 65535 || K <= 0 || K % (wfmt == 2 ? 64 : 32) || K > 16384)
        return fail(COLI_EINVAL, "bad sizes");
    if (!codes || !xq || !S) return fail(COLI_EINVAL, "null pointer");
    if (!aligned16(codes) || !aligned16(xq) || !aligned16(S)) return fail(COLI_EINVAL, "pointers must be 16-byte aligned");
    cudaStream_t s = (cudaStream_t)stream;
    const size_t smem = stage_bytes(1, (int)K);
    dim3 grid((unsigned)std::min<int64_t>((rows + 7) / 8, 1024), (unsigned)T);
    Launch L(nullptr, s, "dbg_block_sums");
    switch (wfmt) {
        case 8: k_dbg_block_sums<8><<<grid, 256, smem, s>>>((const uint8_t *)codes, rows, (int)K, xq, T, S); break;
        case 4: k_dbg_block_sums<4><<<grid, 256, smem, s>>>((const uint8_t *)codes, rows, (int)K, xq, T, S); break;
        default: k_dbg_block_sums<2><<<grid, 256, smem, s>>>((const uint8_t *)codes, rows, (int)K, xq, T, S); break;
    }
    return L.done();
}

coli_status coli_dbg_last_forward(coli_moe *m, int T, int32_t *idx, float *w, int8_t *hq,
                                  float *hd, coli_stream_t stream) {
    g_last_error.clear();
    coli_status st = check_handle(m);
    if (st != COLI_OK) return st;
    if (m->last_T == 0 || T != m->last_T) return fail(COLI_EINVAL, "T=%d does not match the last forward (T=%d)", T, m->last_T);
    cudaStream_t s = (cudaStream_t)stream;
    const auto &c = m->cfg;
    if (idx) COLI_CUDA(cudaMemcpyAsync(idx, m->rw.idx, (size_t)T * c.top_k * 4, cudaMemcpyDeviceToDevice, s), "copy idx");
    if (w) COLI_CUDA(cudaMemcpyAsync(w, m->rw.w, (size_t)T * c.top_k * 4, cudaMemcpyDeviceToDevice, s), "copy w");
    if (hq || hd) {
        const int slots = c.top_k + c.n_shared;
        Launch L(nullptr, s, "dbg_gather_h");
        k_gather_h<<<T * slots, 256, 0, s>>>(m->rw.tok_pair, m->hq, m->hd, T, slots, c.inter, hq, hd);
        return L.done();
    }
    return COLI_OK;
}

}  // extern "C"
