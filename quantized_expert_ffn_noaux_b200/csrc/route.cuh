// route.cuh -- sigmoid noaux_tc router and the batch-union tables.
//
// "Show HN: 遅いコンピュータで GLM 5.2 を実行する", section 実装済みの主な機能:
//   router bullet: DeepSeek-V3-style sigmoid router (noaux_tc with an
//     e_score_correction bias, routed_scaling_factor, shared expert);
//   batch-union bullet: each distinct expert of the batch is read once and
//     applied to every position routed to it.
// Logits are fp64 sums of exact fp32*fp32 products; sigmoid, group scores and
// the selection are fp64; ties go to the lower group / expert index.
#pragma once
#include "common.cuh"

namespace coli {

struct RouteWs {
    double *s, *c;            // [T][E] sigmoid scores and choice scores
    int32_t *idx;             // [T][k]
    float *w;                 // [T][k]
    uint32_t *bitmap;         // [E][wstride] token membership per expert
    int32_t *prefix;          // [E][wstride] popcount prefix per word
    uint32_t *counter;        // last-CTA ticket
    int32_t *n_active;        // [1]
    int32_t *active;          // [E+S] expert id per active slot (ascending, shared last)
    int32_t *off;             // [E+S+1] first pair of each active expert
    int32_t *act_of;          // [E+S] active slot of each expert (-1 if none)
    int32_t *pair_tok;        // [Pmax] token of each pair
    int32_t *pair_slot;       // [Pmax] slot of each pair
    int32_t *tok_pair;        // [T][k+S] pair of each (token, slot); -1: expert not owned here
    int wstride;              // bitmap words per expert
    // expert parallelism: this handle computes routed experts [e_lo, e_hi)
    // and, if own_shared, the shared experts; the batch union holds only those
    int e_lo, e_hi, own_shared;
    __host__ __device__ bool owns(int e) const { return e >= e_lo && e < e_hi; }
    __host__ __device__ int shared_active(int S) const { return own_shared ? S : 0; }
};

// ---------------------------------------------------------------------------
// Logits for few tokens (T <= 8): one warp per expert, lanes stride over H.
template <int NT>
__global__ void k_route_logits_small(const float *__restrict__ x, int T, int H,
                                     const float *__restrict__ Wr, const float *__restrict__ bias,
                                     int E, double *__restrict__ s_out,
                                     double *__restrict__ c_out) {
    const int lane = threadIdx.x & 31;
    const int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (e >= E) return;
    double acc[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t] = 0.0;
    const float4 *w4 = reinterpret_cast<const float4 *>(Wr + (int64_t)e * H);
    const int H4 = H >> 2;
    for (int i = lane; i < H4; i += 32) {
        float4 wv = __ldg(w4 + i);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            if (t < T) {
                float4 xv = __ldg(reinterpret_cast<const float4 *>(x + (int64_t)t * H) + i);
                acc[t] = fma((double)xv.x, (double)wv.x, acc[t]);
                acc[t] = fma((double)xv.y, (double)wv.y, acc[t]);
                acc[t] = fma((double)xv.z, (double)wv.z, acc[t]);
                acc[t] = fma((double)xv.w, (double)wv.w, acc[t]);
            }
        }
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        if (t < T) {
            double l = warp_sum(acc[t]);
            if (lane == 0) {
                double s = 1.0 / (1.0 + exp(-l));
                s_out[(int64_t)t * E + e] = s;
                c_out[(int64_t)t * E + e] = s + (double)bias[e];
            }
        }
    }
}

// Logits for many tokens: 64 tokens x 64 experts per CTA, 256 threads each
// computing a 4 x 4 fp64 tile; K staged through shared memory in fp32, the
// next 32-wide slice loaded into registers while the current one is used.
__global__ void __launch_bounds__(256) k_route_logits_tiled(
    const float *__restrict__ x, int T, int H, const float *__restrict__ Wr,
    const float *__restrict__ bias, int E, double *__restrict__ s_out, double *__restrict__ c_out) {
    constexpr int TM = 64, TN = 64, TK = 32, PER = TM * TK / 256;  // 8 values of x and of W per thread
    __shared__ float xs[TK][TM + 1];
    __shared__ float ws[TK][TN + 1];
    const int tid = threadIdx.x;
    const int t0 = blockIdx.x * TM, e0 = blockIdx.y * TN;
    const int tx = tid & 15, ty = tid >> 4;  // 16 x 16 threads, 4 x 4 each
    double acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
    // element q of this thread in a slice: row r = (tid + 256 q) / TK, column cc = tid % TK
    float nx[PER], nw[PER];
    auto load_slice = [&](int k0) {
#pragma unroll
        for (int q = 0; q < PER; ++q) {
            const int i = tid + 256 * q, r = i / TK, cc = i % TK;
            const int t = t0 + r, e = e0 + r;
            nx[q] = (t < T) ? __ldg(x + (int64_t)t * H + k0 + cc) : 0.0f;
            nw[q] = (e < E) ? __ldg(Wr + (int64_t)e * H + k0 + cc) : 0.0f;
        }
    };
    load_slice(0);
    for (int k0 = 0; k0 < H; k0 += TK) {
#pragma unroll
        for (int q = 0; q < PER; ++q) {
            const int i = tid + 256 * q, r = i / TK, cc = i % TK;
            xs[cc][r] = nx[q];
            ws[cc][r] = nw[q];
        }
        __syncthreads();
        if (k0 + TK < H) load_slice(k0 + TK);  // in flight during this slice's arithmetic
#pragma unroll 4
        for (int kk = 0; kk < TK; ++kk) {
            double xv[4], wv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) xv[i] = (double)xs[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) wv[j] = (double)ws[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fma(xv[i], wv[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int t = t0 + ty * 4 + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int e = e0 + tx * 4 + j;
            if (e >= E) continue;
            double s = 1.0 / (1.0 + exp(-acc[i][j]));
            s_out[(int64_t)t * E + e] = s;
            c_out[(int64_t)t * E + e] = s + (double)bias[e];
        }
    }
}

// ---------------------------------------------------------------------------
// Synchronisation of the 256 threads that run the routing helpers: the whole
// CTA (SyncAll), or the eight consumer warps of a warp-specialised CTA whose
// producer warp does not take part (SyncConsumers, named barrier 1).
struct SyncAll {
    __device__ static void sync() { __syncthreads(); }
};
struct SyncConsumers {
    __device__ static void sync() {
        __syncwarp();
        asm volatile("bar.sync 1, 256;" ::: "memory");
    }
};

// Block-wide exclusive scan of one int per thread (256 participating threads).
template <typename Sync = SyncAll>
__device__ __forceinline__ int block_exscan256(int v, int *tmp /*[8]*/, int &total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) tmp[wid] = inc;
    Sync::sync();
    int base = 0, tot = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int t = tmp[i];
        if (i < wid) base += t;
        tot += t;
    }
    Sync::sync();
    total = tot;
    return base + inc - v;
}

// ---------------------------------------------------------------------------
// Selection of one token by a whole CTA (256 threads), rank based, no serial
// scans:  in-group ranks give each group's two best c (its score); group
// ranks keep the topk_group best groups; the top_k of the kept experts are
// among the min(top_k, E/G) experts ranked first inside their own kept group,
// which are laid out densely (kept-group position x in-group rank), and their
// ranks among those candidates give idx sorted by descending c.  Every
// comparison breaks ties toward the lower index.  Each step is a loop of
// independent shared-memory reads, so it runs at the load issue rate rather
// than at the latency of a dependent chain.
struct SelectSmem {
    double *c;      // [E]
    double *s;      // [E]
    double *candc;  // [E] choice scores of the candidates, in candidate order
    int *grank;     // [E] rank inside its group
    double *top1;   // [G]
    double *top2;   // [G] second best, then the group score
    int *keep;      // [G] 1 if kept, then its position among the kept groups (-1: dropped)
    int *cand;      // [E] expert of each candidate
    int *ncand;     // [1]
    int *sel;       // [32]
    float *w_smem;  // optional [k] copy of the weights (set by the caller)
};

__host__ __device__ inline size_t select_smem_bytes(int E, int G) {
    return (size_t)E * 24 + (size_t)G * 16 + (size_t)E * 8 + (size_t)G * 4 + 4 + 32 * 4 + 64;
}

__device__ inline SelectSmem carve_select(void *base, int E, int G) {
    SelectSmem m;
    char *p = (char *)base;
    m.c = (double *)p;           p += (size_t)E * 8;
    m.s = (double *)p;           p += (size_t)E * 8;
    m.candc = (double *)p;       p += (size_t)E * 8;
    m.top1 = (double *)p;        p += (size_t)G * 8;
    m.top2 = (double *)p;        p += (size_t)G * 8;
    m.grank = (int *)p;          p += (size_t)E * 4;
    m.cand = (int *)p;           p += (size_t)E * 4;
    m.keep = (int *)p;           p += (size_t)G * 4;
    m.ncand = (int *)p;          p += 4;
    m.sel = (int *)p;
    m.w_smem = nullptr;
    return m;
}

// Adaptive expert top-p of one token, by one warp after the top-k
// ("Show HN: 遅いコンピュータで GLM 5.2 を実行する", モデルのダウンロードと実行,
// --topp; reading: keep the selected experts by descending sigmoid score,
// ties to the earlier slot, while the kept scores sum to less than
// p * (sum over the k), the first always; drop the rest; renormalise over the
// kept).  Lane j < k holds slot j's expert ej and score sj; slot_s[0..k) holds
// the same scores in slot order and `total` their slot-order sum.  On return
// ej is -1 for a dropped slot and the result is the slot's weight.  order /
// kept: shared scratch of k ints each.  Every operation on the scores is the
// definition's, in its order (one lane runs the cumulative sum).
__device__ __forceinline__ float warp_top_p(int &ej, double sj, const double *slot_s, int k,
                                            double total, float p, float rsf, int *order,
                                            int *kept) {
    const int lane = threadIdx.x & 31;
    if (lane < k) {
        int r = 0;
        for (int i = 0; i < k; ++i) {
            const double u = slot_s[i];
            r += (int)(u > sj) | ((int)(u == sj) & (int)(i < lane));
        }
        order[r] = lane;
        kept[lane] = 0;
    }
    __syncwarp();
    if (lane == 0) {
        const double cut = (double)p * total;
        double cum = 0.0;
        for (int n = 0; n < k; ++n) {
            const int j = order[n];
            if (n > 0 && !(cum < cut)) break;
            kept[j] = 1;
            cum += slot_s[j];
        }
    }
    __syncwarp();
    double ksum = 0.0;
    for (int i = 0; i < k; ++i)
        if (kept[i]) ksum += slot_s[i];
    const bool keep = lane < k && kept[lane];
    if (!keep) ej = -1;
    return keep ? (float)((sj / ksum) * (double)rsf) : 0.0f;
}

__host__ __device__ inline bool top_p_on(float p) { return p > 0.0f && p < 1.0f; }

// Warp-level selection for the common shape: every group fits one warp
// (E/G <= 32), at most 8 groups, and the kept groups' candidates fit one warp
// (topk_group * min(top_k, E/G) <= 32).  Warp g holds group g, one expert per
// lane; ranks come from branch-free shuffle comparisons (ties: lower index),
// and only three CTA barriers are taken.  Same results as the general path.
__host__ __device__ inline bool select_warp_shape(int E, int G, int gk, int k) {
    const int per = E / G, kk = k < per ? k : per;
    return per <= 32 && G <= 8 && gk * kk <= 32 && k <= 32;
}

template <typename Sync>
__device__ void cta_select_token_warps(const double *c_row, const double *s_row, int E, int G,
                                       int gk, int k, float rsf, const SelectSmem &sm,
                                       int32_t *idx_out, float *w_out, int *idx_smem,
                                       int arrive_bar, int arrive_count, float top_p) {
    const unsigned FULL = 0xffffffffu;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = E / G, kk = k < per ? k : per;
    const int e = warp * per + lane;
    const bool mine = warp < G && lane < per;
    double v = 0.0, sv = 0.0;
    if (mine) {
        v = __ldcg(c_row + e);
        sv = __ldcg(s_row + e);
    }
    int r = 0;
    if (warp < G) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const double u = __shfl_sync(FULL, v, j);
            r += (int)(j < per) & ((int)(u > v) | ((int)(u == v) & (int)(j < lane)));
        }
        // the group's score: its best c plus its second best
        const unsigned m0 = __ballot_sync(FULL, mine && r == 0);
        const unsigned m1 = __ballot_sync(FULL, mine && r == 1);
        const double t1 = __shfl_sync(FULL, v, __ffs(m0) - 1);
        const double t2 = __shfl_sync(FULL, v, m1 ? __ffs(m1) - 1 : 0);
        if (lane == 0) sm.top2[warp] = t1 + (per > 1 ? t2 : 0.0);
    }
    if (arrive_count > 0) {  // this thread's scores (r used them) and async copies have landed
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncwarp();
        asm volatile("bar.arrive %0, %1;" ::"r"(arrive_bar), "r"(arrive_count) : "memory");
    }
    Sync::sync();
    // every warp: the ranks of the G group scores, the kept groups
    const double gsv = lane < G ? sm.top2[lane] : 0.0;
    int grk = 0;
#pragma unroll
    for (int h = 0; h < 8; ++h) {
        const double u = __shfl_sync(FULL, gsv, h);
        grk += (int)(h < G) & ((int)(u > gsv) | ((int)(u == gsv) & (int)(h < lane)));
    }
    const unsigned kept = __ballot_sync(FULL, lane < G && grk < gk);
    if (warp < G && ((kept >> warp) & 1u) && mine && r < kk) {
        const int pos = __popc(kept & ((1u << warp) - 1u)) * kk + r;
        sm.cand[pos] = e;
        sm.candc[pos] = v;
        sm.s[pos] = sv;
    }
    Sync::sync();
    if (warp == 0) {
        const int n = gk * kk;
        const bool has = lane < n;
        const double cv = has ? sm.candc[lane] : 0.0;
        const int ce = has ? sm.cand[lane] : 0;
        const double cs = has ? sm.s[lane] : 0.0;
        int rank = 0;
#pragma unroll 8
        for (int j = 0; j < n; ++j) {  // broadcast reads of every candidate
            const double u = sm.candc[j];
            const int f = sm.cand[j];
            rank += (int)(u > cv) | ((int)(u == cv) & (int)(f < ce));
        }
        // slot j is the candidate of rank j; the weights renormalise s over
        // the slots in slot order, times rsf
        __syncwarp();
        if (has && rank < k) {
            sm.sel[rank] = ce;
            sm.c[rank] = cs;
        }
        __syncwarp();
        double ssum = 0.0;
#pragma unroll 8
        for (int j = 0; j < k; ++j) ssum += sm.c[j];
        int ej = lane < k ? sm.sel[lane] : 0;
        float wj = lane < k ? (float)((sm.c[lane] / ssum) * (double)rsf) : 0.0f;
        if (top_p_on(top_p))
            wj = warp_top_p(ej, lane < k ? sm.c[lane] : 0.0, sm.c, k, ssum, top_p, rsf, sm.cand,
                            sm.grank);
        if (lane < k) {
            if (idx_out) idx_out[lane] = ej;
            if (w_out) w_out[lane] = wj;
            if (idx_smem) idx_smem[lane] = ej;
            if (sm.w_smem) sm.w_smem[lane] = wj;
        }
    }
    Sync::sync();
}

// arrive_bar / arrive_count: if arrive_count > 0, every calling thread
// arrives (bar.arrive) on that named barrier as soon as the token's scores
// and the thread's earlier cp.async copies have landed -- a hook for a warp
// that must not start memory traffic before those loads are done.
template <typename Sync = SyncAll>
__device__ void cta_select_token(const double *c_row, const double *s_row, int E, int G, int gk,
                                 int k, float rsf, const SelectSmem &sm, int32_t *idx_out,
                                 float *w_out, int *idx_smem = nullptr, int arrive_bar = 0,
                                 int arrive_count = 0, float top_p = 0.0f) {
    if (k <= 0 || E <= 0) return;  // a dense layer: nothing to select
    if (select_warp_shape(E, G, gk, k)) {
        cta_select_token_warps<Sync>(c_row, s_row, E, G, gk, k, rsf, sm, idx_out, w_out, idx_smem,
                                     arrive_bar, arrive_count, top_p);
        return;
    }
    const int tid = threadIdx.x, nthr = 256;
    const int per = E / G;
    const int kk = k < per ? k : per;  // candidates one kept group can contribute
    for (int e = tid; e < E; e += nthr) {
        sm.c[e] = __ldcg(c_row + e);
        sm.s[e] = __ldcg(s_row + e);
    }
    Sync::sync();
    if (arrive_count > 0) {  // this thread's scores and async copies have landed
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncwarp();
        asm volatile("bar.arrive %0, %1;" ::"r"(arrive_bar), "r"(arrive_count) : "memory");
    }
    for (int e = tid; e < E; e += nthr) {
        const int g = e / per, g0 = g * per;
        const double v = sm.c[e];
        int r = 0;
#pragma unroll 8
        for (int i = 0; i < per; ++i) {
            const double u = sm.c[g0 + i];
            r += (int)(u > v) | ((int)(u == v) & (int)(g0 + i < e));
        }
        sm.grank[e] = r;
        if (r == 0) sm.top1[g] = v;
        if (r == 1) sm.top2[g] = v;
    }
    Sync::sync();
    for (int g = tid; g < G; g += nthr) sm.top2[g] = sm.top1[g] + (per > 1 ? sm.top2[g] : 0.0);
    Sync::sync();
    for (int g = tid; g < G; g += nthr) {
        const double v = sm.top2[g];
        int r = 0;
#pragma unroll 8
        for (int h = 0; h < G; ++h) {
            const double u = sm.top2[h];
            r += (int)(u > v) | ((int)(u == v) & (int)(h < g));
        }
        sm.keep[g] = r < gk;
    }
    Sync::sync();
    // position of each kept group among the kept groups (index order)
    if (G <= nthr) {
        int kpos = -1;
        if (tid < G) {
            int before = 0;
#pragma unroll 8
            for (int h = 0; h < tid; ++h) before += sm.keep[h];
            kpos = sm.keep[tid] ? before : -1;
        }
        Sync::sync();
        if (tid < G) sm.keep[tid] = kpos;
    } else if (tid == 0) {
        int n = 0;
        for (int g = 0; g < G; ++g) sm.keep[g] = sm.keep[g] ? n++ : -1;
    }
    Sync::sync();
    for (int e = tid; e < E; e += nthr) {
        const int pos = sm.keep[e / per];
        const int r = sm.grank[e];
        if (pos >= 0 && r < kk) {
            sm.cand[pos * kk + r] = e;
            sm.candc[pos * kk + r] = sm.c[e];
        }
    }
    Sync::sync();
    const int n = gk * kk;
    for (int i = tid; i < n; i += nthr) {
        const double v = sm.candc[i];
        const int e = sm.cand[i];
        int r = 0;
#pragma unroll 8
        for (int j = 0; j < n; ++j) {
            const double u = sm.candc[j];
            const int f = sm.cand[j];
            r += (int)(u > v) | ((int)(u == v) & (int)(f < e));
        }
        if (r < k) sm.sel[r] = e;
    }
    Sync::sync();
    if (tid < 32) {
        // weights: s of the selection renormalised (sum in slot order) x rsf
        const int lane = tid;
        const int e = lane < k ? sm.sel[lane] : 0;
        const double sj = lane < k ? sm.s[e] : 0.0;
        double ssum = 0.0;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const double v = __shfl_sync(0xffffffffu, sj, j);
            if (j < k) ssum += v;
        }
        int ej = e;
        float wj = lane < k ? (float)((sj / ssum) * (double)rsf) : 0.0f;
        if (top_p_on(top_p)) {
            if (lane < k) sm.candc[lane] = sj;  // slot-order scores (candc is free by now)
            __syncwarp();
            wj = warp_top_p(ej, sj, sm.candc, k, ssum, top_p, rsf, sm.cand, sm.grank);
        }
        if (lane < k) {
            if (idx_out) idx_out[lane] = ej;
            if (w_out) w_out[lane] = wj;
            if (idx_smem) idx_smem[lane] = ej;
            if (sm.w_smem) sm.w_smem[lane] = wj;
        }
    }
    Sync::sync();
}

// Batch-union tables of a single token, by one warp: the k selected experts
// ascending (one pair each), then the shared experts -- the tables
// cta_union_small builds for T = 1, without its scans over every expert.
__device__ void warp_union_one(RouteWs ws, int E, int S, int k, const int *idx /*smem [k]*/) {
    const int lane = threadIdx.x & 31;
    for (int e = lane; e < E + S; e += 32) ws.act_of[e] = -1;
    __syncwarp();
    // the selected experts this handle owns, ascending
    int nk = 0;
    for (int i = 0; i < k; ++i) nk += ws.owns(idx[i]);
    for (int j = lane; j < k; j += 32) {
        const int e = idx[j];
        if (!ws.owns(e)) {
            ws.tok_pair[j] = -1;
            continue;
        }
        int a = 0;
        for (int i = 0; i < k; ++i) a += ws.owns(idx[i]) && idx[i] < e;
        ws.active[a] = e;
        ws.off[a] = a;
        ws.act_of[e] = a;
        ws.pair_tok[a] = 0;
        ws.pair_slot[a] = j;
        ws.tok_pair[j] = a;
    }
    const int sa = ws.shared_active(S);
    for (int i = lane; i < S; i += 32) {
        if (i >= sa) {
            ws.tok_pair[k + i] = -1;
            continue;
        }
        const int a = nk + i;
        ws.active[a] = E + i;
        ws.off[a] = a;
        ws.act_of[E + i] = a;
        ws.pair_tok[a] = 0;
        ws.pair_slot[a] = k + i;
        ws.tok_pair[k + i] = a;
    }
    if (lane == 0) {
        ws.off[nk + sa] = nk + sa;
        *ws.n_active = nk + sa;
    }
    __syncwarp();
}

// One CTA (256 threads) per token: cta_select_token.  With `do_union`, the
// experts are also marked in the membership bitmap and the last CTA to finish
// builds the batch-union tables.  Dynamic smem: select_smem_bytes(E, G).
__global__ void __launch_bounds__(256) k_route_select(
    RouteWs ws, int T, int E, int S, int G, int gk, int k, float rsf, int32_t *__restrict__ idx_out,
    float *__restrict__ w_out, int do_union, float top_p) {
    extern __shared__ __align__(16) double smem_d[];
    __shared__ int is_last;
    __shared__ int scan_tmp[8];
    const int t = blockIdx.x, tid = threadIdx.x;
    const SelectSmem sm = carve_select(smem_d, E, G);
    cta_select_token(ws.c + (int64_t)t * E, ws.s + (int64_t)t * E, E, G, gk, k, rsf, sm,
                     idx_out + (int64_t)t * k, w_out + (int64_t)t * k, nullptr, 0, 0, top_p);
    double *c_s = sm.c;
    const int *sel = idx_out + (int64_t)t * k;
    if (!do_union) return;
    if (tid < k && ws.owns(sel[tid]))
        atomicOr(ws.bitmap + (int64_t)sel[tid] * ws.wstride + (t >> 5), 1u << (t & 31));
    __threadfence();
    __syncthreads();
    if (tid == 0) is_last = (atomicAdd(ws.counter, 1u) == (unsigned)(gridDim.x - 1));
    __syncthreads();
    if (!is_last) return;
    __threadfence();

    // ---- last CTA: batch-union tables ([HN] batch-union bullet) ----
    const int nw = (T + 31) >> 5;
    int *cnt_s = reinterpret_cast<int *>(c_s);  // reuse: [E]
    for (int e = tid; e < E; e += 256) {
        int c = 0;
        for (int w = 0; w < nw; ++w) {
            ws.prefix[(int64_t)e * ws.wstride + w] = c;
            c += __popc(__ldcg(ws.bitmap + (int64_t)e * ws.wstride + w));
        }
        cnt_s[e] = c;
    }
    __syncthreads();
    // ascending active experts, then the shared experts
    int na_base = 0, pair_base = 0;
    for (int e0 = 0; e0 < E; e0 += 256) {
        int e = e0 + tid;
        int c = (e < E) ? cnt_s[e] : 0;
        int flag = c > 0;
        int ftot, ctot;
        int fpos = block_exscan256(flag, scan_tmp, ftot);
        int cpos = block_exscan256(c, scan_tmp, ctot);
        if (e < E) {
            if (flag) {
                ws.active[na_base + fpos] = e;
                ws.off[na_base + fpos] = pair_base + cpos;
                ws.act_of[e] = na_base + fpos;
            } else {
                ws.act_of[e] = -1;
            }
        }
        na_base += ftot;
        pair_base += ctot;
    }
    const int sa = ws.shared_active(S);
    for (int i = tid; i < S; i += 256) {
        if (i < sa) {
            ws.active[na_base + i] = E + i;
            ws.off[na_base + i] = pair_base + i * T;
            ws.act_of[E + i] = na_base + i;
        } else {
            ws.act_of[E + i] = -1;
        }
    }
    if (tid == 0) {
        ws.off[na_base + sa] = pair_base + sa * T;
        *ws.n_active = na_base + sa;
    }
    __syncthreads();
    const int slots = k + S;
    for (int i = tid; i < T * k; i += 256) {
        int tt = i / k, j = i % k;
        int e = __ldcg(idx_out + i);
        if (!ws.owns(e)) {
            ws.tok_pair[(int64_t)tt * slots + j] = -1;
            continue;
        }
        int64_t wo = (int64_t)e * ws.wstride + (tt >> 5);
        int rank = ws.prefix[wo] + __popc(__ldcg(ws.bitmap + wo) & ((1u << (tt & 31)) - 1u));
        int p = ws.off[ws.act_of[e]] + rank;
        ws.pair_tok[p] = tt;
        ws.pair_slot[p] = j;
        ws.tok_pair[(int64_t)tt * slots + j] = p;
    }
    for (int i = tid; i < T * S; i += 256) {
        int tt = i % T, sh = i / T;
        if (sh >= sa) {
            ws.tok_pair[(int64_t)tt * slots + k + sh] = -1;
            continue;
        }
        int p = ws.off[na_base + sh] + tt;
        ws.pair_tok[p] = tt;
        ws.pair_slot[p] = k + sh;
        ws.tok_pair[(int64_t)tt * slots + k + sh] = p;
    }
    __syncthreads();
    for (int i = tid; i < E * nw; i += 256) ws.bitmap[(int64_t)(i / nw) * ws.wstride + (i % nw)] = 0u;
    if (tid == 0) *ws.counter = 0u;
}


// Batch-union tables for few tokens (T * k <= 256), built by one CTA from
// idx [T][k]: active experts ascending (shared experts last), each expert's
// tokens in token order.
template <typename Sync = SyncAll>
__device__ void cta_union_small(RouteWs ws, int T, int E, int S, int k,
                                int *cnt /*smem [E]*/, const int *idx /*smem [T*k]*/,
                                int *scan_tmp /*smem [8]*/) {
    const int tid = threadIdx.x;
    for (int e = tid; e < E; e += 256) {
        int c = 0;
        if (ws.owns(e))
            for (int i = 0; i < T * k; ++i) c += (idx[i] == e);
        cnt[e] = c;
    }
    // slots of experts this handle does not own stay -1
    for (int i = tid; i < T * (k + S); i += 256) ws.tok_pair[i] = -1;
    Sync::sync();
    int na_base = 0, pair_base = 0;
    for (int e0 = 0; e0 < E; e0 += 256) {
        const int e = e0 + tid;
        const int c = (e < E) ? cnt[e] : 0;
        const int flag = c > 0;
        int ftot, ctot;
        const int fpos = block_exscan256<Sync>(flag, scan_tmp, ftot);
        const int cpos = block_exscan256<Sync>(c, scan_tmp, ctot);
        if (e < E) {
            if (flag) {
                const int a = na_base + fpos;
                int p = pair_base + cpos;
                ws.active[a] = e;
                ws.off[a] = p;
                ws.act_of[e] = a;
                for (int i = 0; i < T * k; ++i)
                    if (idx[i] == e) {
                        const int t = i / k, j = i % k;
                        ws.pair_tok[p] = t;
                        ws.pair_slot[p] = j;
                        ws.tok_pair[t * (k + S) + j] = p;
                        ++p;
                    }
            } else {
                ws.act_of[e] = -1;
            }
        }
        na_base += ftot;
        pair_base += ctot;
    }
    const int sa = ws.shared_active(S);
    for (int i = tid; i < S; i += 256) {
        if (i >= sa) {
            ws.act_of[E + i] = -1;
            continue;
        }
        const int a = na_base + i;
        ws.active[a] = E + i;
        ws.off[a] = pair_base + i * T;
        ws.act_of[E + i] = a;
        for (int t = 0; t < T; ++t) {
            const int p = pair_base + i * T + t;
            ws.pair_tok[p] = t;
            ws.pair_slot[p] = k + i;
            ws.tok_pair[t * (k + S) + k + i] = p;
        }
    }
    if (tid == 0) {
        ws.off[na_base + sa] = pair_base + sa * T;
        *ws.n_active = na_base + sa;
    }
}

// Router for few tokens (T <= NT), one kernel: CTA e computes the fp64 logit
// of expert e for every token, all CTAs share the Q8_0 of x (natural codes
// and the records the expert kernels stage), and the last CTA to finish
// selects every token's experts and builds the batch-union tables.
// blockDim.x == 256; dynamic smem = select_smem_bytes(E, G) + 4*E.
template <int NT, int BITS>
__global__ void __launch_bounds__(256) k_router_small(
    const float *__restrict__ x, int T, int H, const float *__restrict__ Wr,
    const float *__restrict__ bias, int E, int S, int G, int gk, int k, float rsf, RouteWs ws,
    uint8_t *__restrict__ xrec, int8_t *__restrict__ xq, float *__restrict__ xd,
    int do_union, int32_t *__restrict__ idx_out, float *__restrict__ w_out, float top_p) {
    extern __shared__ __align__(16) uint8_t smem_r[];
    __shared__ double red[8][NT];
    __shared__ int is_last;
    __shared__ int scan_tmp[8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int e = blockIdx.x;
    // ---- logit of expert e for every token (fp64 sum of exact products)
    {
        double acc[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[t] = 0.0;
        const float4 *w4 = reinterpret_cast<const float4 *>(Wr + (int64_t)e * H);
        for (int i = tid; i < H / 4; i += 256) {
            const float4 wv = __ldg(w4 + i);
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                if (t < T) {
                    const float4 xv = __ldg(reinterpret_cast<const float4 *>(x + (int64_t)t * H) + i);
                    acc[t] = fma((double)xv.x, (double)wv.x, acc[t]);
                    acc[t] = fma((double)xv.y, (double)wv.y, acc[t]);
                    acc[t] = fma((double)xv.z, (double)wv.z, acc[t]);
                    acc[t] = fma((double)xv.w, (double)wv.w, acc[t]);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const double v = warp_sum(acc[t]);
            if (lane == 0) red[warp][t] = v;
        }
        __syncthreads();
        if (tid < T) {
            double l = 0.0;
            for (int w = 0; w < 8; ++w) l += red[w][tid];
            const double sg = 1.0 / (1.0 + exp(-l));
            ws.s[(int64_t)tid * E + e] = sg;
            ws.c[(int64_t)tid * E + e] = sg + (double)bias[e];
        }
    }
    // ---- Q8_0(x): warps of all CTAs share the T * H/32 blocks
    if (do_union) {
        const int nb = H / COLI_QBLK;
        const int rb = rec_bytes(H);
        for (int blk = blockIdx.x * 8 + warp; blk < T * nb; blk += gridDim.x * 8) {
            const int t = blk / nb, b = blk % nb;
            const float v = __ldg(x + (int64_t)t * H + b * COLI_QBLK + lane);
            q8_block_to_record<BITS>(v, b, H, xrec + (size_t)t * rb, xq + (int64_t)t * H,
                                     xd + (int64_t)t * nb);
        }
    }
    // ---- last CTA: selection and the union tables
    __threadfence();
    __syncthreads();
    if (tid == 0) is_last = (atomicAdd(ws.counter, 1u) == (unsigned)(gridDim.x - 1));
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    const SelectSmem sm = carve_select(smem_r, E, G);
    int32_t *idx_dst = do_union ? ws.idx : idx_out;
    float *w_dst = do_union ? ws.w : w_out;
    int *cnt = reinterpret_cast<int *>(smem_r + select_smem_bytes(E, G));
    int *idx_s = cnt + E;
    for (int t = 0; t < T; ++t)
        cta_select_token(ws.c + (int64_t)t * E, ws.s + (int64_t)t * E, E, G, gk, k, rsf, sm,
                         idx_dst + t * k, w_dst + t * k, idx_s + t * k, 0, 0, top_p);
    if (do_union) cta_union_small(ws, T, E, S, k, cnt, idx_s, scan_tmp);
    __syncthreads();
    if (tid == 0) *ws.counter = 0u;
}

// Q8_0 of x for many tokens: natural codes and scales plus the records.
template <int BITS>
__global__ void k_x_prep(const float *__restrict__ x, int T, int H, uint8_t *__restrict__ xrec,
                         int8_t *__restrict__ xq, float *__restrict__ xd) {
    const int lane = threadIdx.x & 31;
    const int nb = H / COLI_QBLK, rb = rec_bytes(H);
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t blk = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
         blk < (int64_t)T * nb; blk += nwarps) {
        const int t = (int)(blk / nb), b = (int)(blk % nb);
        const float v = __ldg(x + (int64_t)t * H + b * COLI_QBLK + lane);
        q8_block_to_record<BITS>(v, b, H, xrec + (size_t)t * rb, xq + (int64_t)t * H,
                                 xd + (int64_t)t * nb);
    }
}

}  // namespace coli
