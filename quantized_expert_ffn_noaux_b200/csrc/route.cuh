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
    int32_t *tok_pair;        // [T][k+S] pair of each (token, slot)
    int wstride;              // bitmap words per expert
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
// computing a 4 x 4 fp64 tile; K staged through shared memory in fp32.
__global__ void __launch_bounds__(256) k_route_logits_tiled(
    const float *__restrict__ x, int T, int H, const float *__restrict__ Wr,
    const float *__restrict__ bias, int E, double *__restrict__ s_out, double *__restrict__ c_out) {
    constexpr int TM = 64, TN = 64, TK = 32;
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
    for (int k0 = 0; k0 < H; k0 += TK) {
        // 64 rows x 32 cols of x and of W: 2048 floats each, 8 per thread
        for (int i = tid; i < TM * TK; i += 256) {
            int r = i / TK, cc = i % TK;
            int t = t0 + r, e = e0 + r;
            xs[cc][r] = (t < T) ? __ldg(x + (int64_t)t * H + k0 + cc) : 0.0f;
            ws[cc][r] = (e < E) ? __ldg(Wr + (int64_t)e * H + k0 + cc) : 0.0f;
        }
        __syncthreads();
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
// Block-wide exclusive scan of one int per thread (blockDim.x == 256).
__device__ __forceinline__ int block_exscan256(int v, int *tmp /*[8]*/, int &total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) tmp[wid] = inc;
    __syncthreads();
    int base = 0, tot = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int t = tmp[i];
        if (i < wid) base += t;
        tot += t;
    }
    __syncthreads();
    total = tot;
    return base + inc - v;
}

// One CTA (256 threads) per token: group scores, group and expert ranks,
// renormalised weights.  With `do_union`, the experts are also marked in the
// membership bitmap and the last CTA to finish builds the batch-union tables.
__global__ void __launch_bounds__(256) k_route_select(
    RouteWs ws, int T, int E, int S, int G, int gk, int k, float rsf, int32_t *__restrict__ idx_out,
    float *__restrict__ w_out, int do_union) {
    extern __shared__ double smem_d[];
    double *c_s = smem_d;                 // [E]
    double *gscore = c_s + E;             // [G]
    int *keep = (int *)(gscore + G);      // [G]
    int *sel = keep + G;                  // [k]
    __shared__ int is_last;
    __shared__ int scan_tmp[8];
    const int t = blockIdx.x, tid = threadIdx.x;
    const int per = E / G;
    const double *c_t = ws.c + (int64_t)t * E;
    for (int e = tid; e < E; e += 256) c_s[e] = c_t[e];
    __syncthreads();
    for (int g = tid; g < G; g += 256) {
        int b1 = -1, b2 = -1;
        for (int i = 0; i < per; ++i) {
            int e = g * per + i;
            if (b1 < 0 || c_s[e] > c_s[b1]) b1 = e;
        }
        for (int i = 0; i < per; ++i) {
            int e = g * per + i;
            if (e == b1) continue;
            if (b2 < 0 || c_s[e] > c_s[b2]) b2 = e;
        }
        gscore[g] = c_s[b1] + (b2 >= 0 ? c_s[b2] : 0.0);
    }
    __syncthreads();
    for (int g = tid; g < G; g += 256) {
        int rank = 0;
        double v = gscore[g];
        for (int h = 0; h < G; ++h) {
            double u = gscore[h];
            rank += (u > v) || (u == v && h < g);
        }
        keep[g] = rank < gk;
    }
    __syncthreads();
    for (int e = tid; e < E; e += 256) {
        if (!keep[e / per]) continue;
        int rank = 0;
        double v = c_s[e];
        for (int f = 0; f < E; ++f) {
            if (!keep[f / per]) continue;
            double u = c_s[f];
            rank += (u > v) || (u == v && f < e);
        }
        if (rank < k) sel[rank] = e;
    }
    __syncthreads();
    if (tid == 0) {
        const double *s_t = ws.s + (int64_t)t * E;
        double ssum = 0.0;
        for (int j = 0; j < k; ++j) ssum += s_t[sel[j]];
        for (int j = 0; j < k; ++j) {
            int e = sel[j];
            float wj = (float)((s_t[e] / ssum) * (double)rsf);
            idx_out[(int64_t)t * k + j] = e;
            w_out[(int64_t)t * k + j] = wj;
        }
    }
    if (!do_union) return;
    if (tid < k) atomicOr(ws.bitmap + (int64_t)sel[tid] * ws.wstride + (t >> 5), 1u << (t & 31));
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
    for (int i = tid; i < S; i += 256) {
        ws.active[na_base + i] = E + i;
        ws.off[na_base + i] = pair_base + i * T;
        ws.act_of[E + i] = na_base + i;
    }
    if (tid == 0) {
        ws.off[na_base + S] = pair_base + S * T;
        *ws.n_active = na_base + S;
    }
    __syncthreads();
    const int slots = k + S;
    for (int i = tid; i < T * k; i += 256) {
        int tt = i / k, j = i % k;
        int e = __ldcg(idx_out + i);
        int64_t wo = (int64_t)e * ws.wstride + (tt >> 5);
        int rank = ws.prefix[wo] + __popc(__ldcg(ws.bitmap + wo) & ((1u << (tt & 31)) - 1u));
        int p = ws.off[ws.act_of[e]] + rank;
        ws.pair_tok[p] = tt;
        ws.pair_slot[p] = j;
        ws.tok_pair[(int64_t)tt * slots + j] = p;
    }
    for (int i = tid; i < T * S; i += 256) {
        int tt = i % T, sh = i / T;
        int p = ws.off[na_base + sh] + tt;
        ws.pair_tok[p] = tt;
        ws.pair_slot[p] = k + sh;
        ws.tok_pair[(int64_t)tt * slots + k + sh] = p;
    }
    __syncthreads();
    for (int i = tid; i < E * nw; i += 256) ws.bitmap[(int64_t)(i / nw) * ws.wstride + (i % nw)] = 0u;
    if (tid == 0) *ws.counter = 0u;
}

}  // namespace coli
