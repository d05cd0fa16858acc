// expert.cuh -- batched integer-dot kernels of the routed and shared experts.
//
// "Show HN: 遅いコンピュータで GLM 5.2 を実行する", section 実装済みの主な機能:
//   integer-dot bullet  -- int8 activation codes (Q8_0) times weight codes,
//                          integer sums per 32-block, then scaled;
//   quantisation bullet -- int8 / packed int4 / packed int2 weights with
//                          per-row scales, dequantised on use;
//   batch-union bullet  -- every distinct expert is read once per forward and
//                          applied to all tokens routed to it.
// "Comment exécuter un réseau de neurones ..." (devtrends.cc), section
// "Comment fonctionne le moteur": an expert is gate, up and down matrices.
//
// Weight rows are streamed from HBM once per work item with 16-byte
// non-allocating loads; the tokens of the item's expert are staged in shared
// memory in the dp4a-ready layout of common.cuh, and every weight vector is
// reused for all staged tokens from registers.
#pragma once
#include "common.cuh"
#include "route.cuh"

namespace coli {

struct QMatDev {
    const uint8_t *codes;
    const float *scales;
};
struct ExpertDev {
    QMatDev gate, up, down;
};

// Shared-memory footprint of `nt` staged activation rows of length K.
__host__ __device__ inline size_t stage_bytes(int nt, int K) {
    return (size_t)nt * (size_t)K + (size_t)nt * (size_t)(K / COLI_QBLK) * 8;
}

// Stage activation rows into shared memory.  Row i (< nt) is source row
// src_row(i) of codes q [*][K] and scales d [*][K/32].
//   planes: [nt][K] bytes, xs: [nt][K/32] int block code sums, xd: [nt][K/32].
template <int BITS, typename RowFn>
__device__ __forceinline__ void stage_rows(const int8_t *__restrict__ q,
                                           const float *__restrict__ d, int K, int nt,
                                           RowFn src_row, uint8_t *planes, int *xs, float *xd) {
    constexpr int ELEMS = Fmt<BITS>::ELEMS;
    const int V = K * BITS / 128;
    const int words = K / 4;  // 32-bit words per staged row
    const int nb = K / COLI_QBLK;
    for (int i = threadIdx.x; i < nt * words; i += blockDim.x) {
        const int r = i / words, wd = i % words;
        const int64_t src = (int64_t)src_row(r) * K;
        const int ob = wd * 4;                 // byte offset in the staged row
        const int plane = ob / (V * 16);
        const int inner = ob % (V * 16);
        const int v = inner / 16;
        const int pos = plane * 16 + (inner % 16);
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            int el = v * ELEMS + stage_src<BITS>(pos + b);
            word |= (uint32_t)(uint8_t)q[src + el] << (8 * b);
        }
        reinterpret_cast<uint32_t *>(planes + (size_t)r * K)[wd] = word;
    }
    for (int i = threadIdx.x; i < nt * nb; i += blockDim.x) {
        const int r = i / nb, b = i % nb;
        const int64_t src = (int64_t)src_row(r);
        const int8_t *qb = q + src * K + b * COLI_QBLK;
        int sum = 0;
#pragma unroll
        for (int j = 0; j < COLI_QBLK; j += 4) {
            int w4 = *reinterpret_cast<const int *>(qb + j);
            sum = dp4a_ss(w4, 0x01010101, sum);
        }
        xs[r * nb + b] = sum;
        xd[r * nb + b] = d[src * (K / COLI_QBLK) + b];
    }
}

// fp64 dot of one weight row (V uint4 vectors, lanes stride by 32) with the
// `nt` staged rows; returns the full sums in every lane.
template <int BITS, int NT, int VPL>
__device__ __forceinline__ void row_dot(const uint4 *__restrict__ row, int V, int K, int nt,
                                        const uint8_t *planes, const int *xs, const float *xd,
                                        double (&acc)[NT]) {
    const int lane = threadIdx.x & 31;
    const int nb = K / COLI_QBLK;
    uint4 wv[VPL];
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
        int v = lane + 32 * j;
        wv[j] = (v < V) ? ldg_stream(row + v) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < NT; ++i) acc[i] = 0.0;
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
        int v = lane + 32 * j;
        if (v < V) {
#pragma unroll
            for (int i = 0; i < NT; ++i) {
                if (i < nt) {
                    const uint4 *act = reinterpret_cast<const uint4 *>(planes + (size_t)i * K) + v;
                    int s0, s1;
                    vec_dot<BITS>(wv[j], act, V, s0, s1);
                    acc[i] = vec_promote<BITS>(v, s0, s1, xs + i * nb, xd + i * nb, acc[i]);
                }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < NT; ++i)
        if (i < nt) acc[i] = warp_sum(acc[i]);
}

// Generic row loop for rows longer than VPL*32 vectors.
template <int BITS, int NT>
__device__ __forceinline__ void row_dot_loop(const uint4 *__restrict__ row, int V, int K, int nt,
                                             const uint8_t *planes, const int *xs,
                                             const float *xd, double (&acc)[NT]) {
    const int lane = threadIdx.x & 31;
    const int nb = K / COLI_QBLK;
#pragma unroll
    for (int i = 0; i < NT; ++i) acc[i] = 0.0;
    for (int v = lane; v < V; v += 32) {
        uint4 w = ldg_stream(row + v);
#pragma unroll
        for (int i = 0; i < NT; ++i) {
            if (i < nt) {
                const uint4 *act = reinterpret_cast<const uint4 *>(planes + (size_t)i * K) + v;
                int s0, s1;
                vec_dot<BITS>(w, act, V, s0, s1);
                acc[i] = vec_promote<BITS>(v, s0, s1, xs + i * nb, xd + i * nb, acc[i]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < NT; ++i)
        if (i < nt) acc[i] = warp_sum(acc[i]);
}

template <int BITS, int NT, int VPL>
__device__ __forceinline__ void any_row_dot(const uint4 *row, int V, int K, int nt,
                                            const uint8_t *planes, const int *xs, const float *xd,
                                            double (&acc)[NT]) {
    if (VPL > 0)
        row_dot<BITS, NT, (VPL > 0 ? VPL : 1)>(row, V, K, nt, planes, xs, xd, acc);
    else
        row_dot_loop<BITS, NT>(row, V, K, nt, planes, xs, xd, acc);
}

constexpr int ROWS_PER_ITEM = 32;  // one Q8_0 block of the intermediate h
constexpr int GROUP_WARPS = 8;
constexpr int GROUP_NT = 8;        // tokens staged per pass

// Gate/up of every (active expert, 32-row chunk) item, fused with SwiGLU and
// Q8_0(h):  g = int_dot(gate), u = int_dot(up), h = (float)(g/(1+e^-g) * u)
// in fp64, then the 32 h values of the chunk form one Q8_0 block.
// Persistent grid: CTAs stride over the n_active * (I/32) items.
template <int BITS, int VPL>
__global__ void __launch_bounds__(256) k_gateup(RouteWs ws, const ExpertDev *__restrict__ experts,
                                                const int8_t *__restrict__ xq,
                                                const float *__restrict__ xd, int H, int I,
                                                int8_t *__restrict__ hq, float *__restrict__ hd) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *planes = smem;
    int *xs = reinterpret_cast<int *>(smem + (size_t)GROUP_NT * H);
    float *xdd = reinterpret_cast<float *>(xs + GROUP_NT * (H / COLI_QBLK));
    float *gu = xdd + GROUP_NT * (H / COLI_QBLK);  // [2][32][GROUP_NT]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nchunk = I / ROWS_PER_ITEM;
    const int n_items = *ws.n_active * nchunk;
    const int V = H * BITS / 128;
    const int64_t rowbytes = (int64_t)H * BITS / 8;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int a = item / nchunk, c = item % nchunk;
        const int e = ws.active[a];
        const int p0 = ws.off[a], ne = ws.off[a + 1] - p0;
        const ExpertDev ex = experts[e];
        for (int tc = 0; tc < ne; tc += GROUP_NT) {
            const int nt = min(GROUP_NT, ne - tc);
            __syncthreads();
            stage_rows<BITS>(xq, xd, H, nt, [&](int i) { return ws.pair_tok[p0 + tc + i]; },
                             planes, xs, xdd);
            __syncthreads();
            for (int rr = warp; rr < 2 * ROWS_PER_ITEM; rr += GROUP_WARPS) {
                const int mat = rr / ROWS_PER_ITEM, r = c * ROWS_PER_ITEM + rr % ROWS_PER_ITEM;
                const QMatDev M = mat == 0 ? ex.gate : ex.up;
                const uint4 *row = reinterpret_cast<const uint4 *>(M.codes + r * rowbytes);
                double acc[GROUP_NT];
                any_row_dot<BITS, GROUP_NT, VPL>(row, V, H, nt, planes, xs, xdd, acc);
                if (lane == 0) {
                    const double sc = (double)M.scales[r];
#pragma unroll
                    for (int i = 0; i < GROUP_NT; ++i)
                        if (i < nt) gu[(mat * ROWS_PER_ITEM + rr % ROWS_PER_ITEM) * GROUP_NT + i] =
                                        (float)(acc[i] * sc);
                }
            }
            __syncthreads();
            // SwiGLU + Q8_0(h): warp i handles staged token i, lane = row in chunk
            for (int i = warp; i < nt; i += GROUP_WARPS) {
                const float g = gu[(0 * ROWS_PER_ITEM + lane) * GROUP_NT + i];
                const float u = gu[(1 * ROWS_PER_ITEM + lane) * GROUP_NT + i];
                const double gd = (double)g;
                const float h = (float)((gd / (1.0 + exp(-gd))) * (double)u);
                float dh;
                const int code = q8_lane(h, dh);
                const int p = p0 + tc + i;
                hq[(int64_t)p * I + c * ROWS_PER_ITEM + lane] = (int8_t)code;
                if (lane == 0) hd[(int64_t)p * (I / COLI_QBLK) + c] = dh;
            }
        }
    }
}

// Down projection for many tokens: e[p][r] = int_dot(down, Q8_0(h_p)) as fp32,
// one item per (active expert, 32-row chunk of H).
template <int BITS, int VPL>
__global__ void __launch_bounds__(256) k_down_grouped(RouteWs ws,
                                                      const ExpertDev *__restrict__ experts,
                                                      const int8_t *__restrict__ hq,
                                                      const float *__restrict__ hd, int H, int I,
                                                      float *__restrict__ e_pairs) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *planes = smem;
    int *xs = reinterpret_cast<int *>(smem + (size_t)GROUP_NT * I);
    float *xdd = reinterpret_cast<float *>(xs + GROUP_NT * (I / COLI_QBLK));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nchunk = H / ROWS_PER_ITEM;
    const int n_items = *ws.n_active * nchunk;
    const int V = I * BITS / 128;
    const int64_t rowbytes = (int64_t)I * BITS / 8;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int a = item / nchunk, c = item % nchunk;
        const int e = ws.active[a];
        const int p0 = ws.off[a], ne = ws.off[a + 1] - p0;
        const QMatDev M = experts[e].down;
        for (int tc = 0; tc < ne; tc += GROUP_NT) {
            const int nt = min(GROUP_NT, ne - tc);
            __syncthreads();
            stage_rows<BITS>(hq, hd, I, nt, [&](int i) { return p0 + tc + i; }, planes, xs, xdd);
            __syncthreads();
            for (int rr = warp; rr < ROWS_PER_ITEM; rr += GROUP_WARPS) {
                const int r = c * ROWS_PER_ITEM + rr;
                const uint4 *row = reinterpret_cast<const uint4 *>(M.codes + r * rowbytes);
                double acc[GROUP_NT];
                any_row_dot<BITS, GROUP_NT, VPL>(row, V, I, nt, planes, xs, xdd, acc);
                if (lane == 0) {
                    const double sc = (double)M.scales[r];
#pragma unroll
                    for (int i = 0; i < GROUP_NT; ++i)
                        if (i < nt) e_pairs[(int64_t)(p0 + tc + i) * H + r] = (float)(acc[i] * sc);
                }
            }
        }
    }
}

// Combine for many tokens: out[t][r] = fp64 sum, shared experts first, then
// routed slots in order, of weight * e (weight 1 for shared experts).
__global__ void k_combine(RouteWs ws, const float *__restrict__ e_pairs, int T, int H, int k,
                          int S, float *__restrict__ out, double *__restrict__ out_partial) {
    const int64_t n = (int64_t)T * H;
    const int slots = k + S;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int t = (int)(i / H), r = (int)(i % H);
        double acc = 0.0;
        for (int jj = 0; jj < slots; ++jj) {
            const int j = jj < S ? k + jj : jj - S;
            const int p = ws.tok_pair[(int64_t)t * slots + j];
            if (p < 0) continue;  // an expert another handle computes
            const double ev = (double)e_pairs[(int64_t)p * H + r];
            if (j < k)
                acc = fma((double)ws.w[(int64_t)t * k + j], ev, acc);
            else
                acc += ev;
        }
        if (out_partial)
            out_partial[i] = acc;
        else
            out[i] = (float)acc;
    }
}

// Down projection + combine for few tokens (decode / verification batches):
// every CTA stages Q8_0(h) of all pairs once; a warp owns 4 output rows and
// walks the active experts in order, then combines each token's slots in the
// fixed order (shared first, then routed slots) in fp64 -- no atomics.
constexpr int DOWN_ROWS = 4;
template <int BITS, int VPL>
__global__ void __launch_bounds__(256) k_down_combine(RouteWs ws,
                                                      const ExpertDev *__restrict__ experts,
                                                      const int8_t *__restrict__ hq,
                                                      const float *__restrict__ hd, int T, int H,
                                                      int I, int k, int S,
                                                      float *__restrict__ out,
                                                      double *__restrict__ out_partial) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_active = *ws.n_active;
    const int n_pairs = ws.off[n_active];
    const int nb = I / COLI_QBLK;
    uint8_t *planes = smem;
    int *xs = reinterpret_cast<int *>(smem + (size_t)n_pairs * I);
    float *xdd = reinterpret_cast<float *>(xs + n_pairs * nb);
    double *ep = reinterpret_cast<double *>(xdd + n_pairs * nb);  // [8 warps][n_pairs][DOWN_ROWS]
    ep += (size_t)warp * n_pairs * DOWN_ROWS;
    // 8-byte alignment of ep: n_pairs*I is a multiple of 32 and nb*8 bytes too.
    stage_rows<BITS>(hq, hd, I, n_pairs, [](int i) { return i; }, planes, xs, xdd);
    __syncthreads();
    const int V = I * BITS / 128;
    const int64_t rowbytes = (int64_t)I * BITS / 8;
    const int slots = k + S;
    const int ngroups = H / DOWN_ROWS;
    for (int g = blockIdx.x * GROUP_WARPS + warp; g < ngroups; g += gridDim.x * GROUP_WARPS) {
        const int r0 = g * DOWN_ROWS;
        for (int a = 0; a < n_active; ++a) {
            const int e = ws.active[a];
            const int p0 = ws.off[a], ne = ws.off[a + 1] - p0;
            const QMatDev M = experts[e].down;
            uint4 wv[DOWN_ROWS][VPL > 0 ? VPL : 1];
            if (VPL > 0) {
#pragma unroll
                for (int rr = 0; rr < DOWN_ROWS; ++rr)
#pragma unroll
                    for (int j = 0; j < (VPL > 0 ? VPL : 1); ++j) {
                        int v = lane + 32 * j;
                        wv[rr][j] = (v < V) ? ldg_stream(reinterpret_cast<const uint4 *>(
                                                  M.codes + (r0 + rr) * rowbytes) + v)
                                            : make_uint4(0, 0, 0, 0);
                    }
            }
            for (int i = 0; i < ne; ++i) {
                const int p = p0 + i;
                const uint8_t *pl = planes + (size_t)p * I;
                double acc[DOWN_ROWS];
#pragma unroll
                for (int rr = 0; rr < DOWN_ROWS; ++rr) acc[rr] = 0.0;
                if (VPL > 0) {
#pragma unroll
                    for (int j = 0; j < (VPL > 0 ? VPL : 1); ++j) {
                        int v = lane + 32 * j;
                        if (v < V) {
#pragma unroll
                            for (int rr = 0; rr < DOWN_ROWS; ++rr) {
                                int s0, s1;
                                vec_dot<BITS>(wv[rr][j], reinterpret_cast<const uint4 *>(pl) + v,
                                              V, s0, s1);
                                acc[rr] = vec_promote<BITS>(v, s0, s1, xs + p * nb, xdd + p * nb,
                                                            acc[rr]);
                            }
                        }
                    }
                } else {
                    for (int v = lane; v < V; v += 32) {
#pragma unroll
                        for (int rr = 0; rr < DOWN_ROWS; ++rr) {
                            uint4 w = ldg_stream(
                                reinterpret_cast<const uint4 *>(M.codes + (r0 + rr) * rowbytes) + v);
                            int s0, s1;
                            vec_dot<BITS>(w, reinterpret_cast<const uint4 *>(pl) + v, V, s0, s1);
                            acc[rr] = vec_promote<BITS>(v, s0, s1, xs + p * nb, xdd + p * nb,
                                                        acc[rr]);
                        }
                    }
                }
#pragma unroll
                for (int rr = 0; rr < DOWN_ROWS; ++rr) {
                    double tot = warp_sum(acc[rr]);
                    if (lane == 0)
                        ep[(size_t)p * DOWN_ROWS + rr] =
                            (double)(float)(tot * (double)M.scales[r0 + rr]);
                }
            }
        }
        __syncwarp();
        // combine: lane handles (token, row) pairs
        for (int q = lane; q < T * DOWN_ROWS; q += 32) {
            const int t = q / DOWN_ROWS, rr = q % DOWN_ROWS;
            double acc = 0.0;
            for (int jj = 0; jj < slots; ++jj) {
                const int j = jj < S ? k + jj : jj - S;
                const int p = ws.tok_pair[(int64_t)t * slots + j];
                if (p < 0) continue;  // an expert another handle computes
                const double ev = ep[(size_t)p * DOWN_ROWS + rr];
                if (j < k)
                    acc = fma((double)ws.w[(int64_t)t * k + j], ev, acc);
                else
                    acc += ev;
            }
            if (out_partial)
                out_partial[(int64_t)t * H + r0 + rr] = acc;
            else
                out[(int64_t)t * H + r0 + rr] = (float)acc;
        }
        __syncwarp();
    }
}

// ===========================================================================
// Few-token (decode / verification) kernels: weight rows stream through a
// shared-memory ring with cp.async.bulk copies issued by one producer thread
// and completed on mbarriers; eight consumer warps run the integer dots out
// of shared memory (nine warps in all, so no SM sub-partition holds more than
// three and each thread may use up to 168 registers).  One CTA per SM, persistent.  Every wait is bounded: on a
// timeout the kernel records COLI_ETIMEOUT in *err, drains its own copies and
// returns.
constexpr int PIPE_CONSUMERS = 8;
constexpr int PIPE_THREADS = 32 * (PIPE_CONSUMERS + 1);
// the decode kernel adds an epilogue warp and an h-fetch warp: 8 consumers,
// producer, epilogue, h fetch
constexpr int DECODE_THREADS = 32 * (PIPE_CONSUMERS + 3);
constexpr int PIPE_STAGE_MAX = 24 * 1024;  // bytes of weights per ring stage (at most)
constexpr int PIPE_MAX_STAGES = 8;
constexpr int PIPE_MAX_TOK = 8;            // tokens per expert on the few-token path
constexpr int PIPE_PASS_TOK = 4;           // tokens per pass over a staged weight row

struct PipeBars {
    uint64_t full[PIPE_MAX_STAGES];
    uint64_t empty[PIPE_MAX_STAGES];
    uint64_t act;
    int abort;
};

__host__ __device__ inline size_t pipe_hdr_bytes() { return (sizeof(PipeBars) + 8 + 64 + 127) & ~(size_t)127; }
__host__ __device__ inline size_t align128(size_t x) { return (x + 127) & ~(size_t)127; }

// Gate/up rows per stage: a power of two dividing 32 with R * rowbytes <= 24 KB.
__host__ __device__ inline int pipe_rows_per_stage(int rowbytes) {
    int r = 32;
    while (r > 1 && r * rowbytes > PIPE_STAGE_MAX) r >>= 1;
    return r;
}

// Producer-side drain after an error: wait (bounded) for every copy still in
// flight on the ring so no copy lands in shared memory after the CTA exits.
__device__ inline void pipe_drain(PipeBars *bars, int ns, long long issued, long long consumed,
                                  int *err) {
    for (long long s = consumed; s < issued; ++s)
        mbar_wait(&bars->full[s % ns], (uint32_t)((s / ns) & 1), err);
}

__device__ inline void pipe_init(PipeBars *bars, int ns) {
    if (threadIdx.x == 0) {
        for (int i = 0; i < ns; ++i) {
            mbar_init(&bars->full[i], 1);
            mbar_init(&bars->empty[i], PIPE_CONSUMERS);
        }
        mbar_init(&bars->act, 1);
        bars->abort = 0;
        fence_mbar_init();
    }
}

// Lane partial dot products of one row slice [v_lo, v_hi) (lanes stride by
// 32 vectors) with NT activation records; unrolled by two for ILP.
template <int BITS, int NT>
__device__ __forceinline__ void slice_dot(const uint4 *__restrict__ wrow, int v_lo, int v_hi, int V,
                                          int K, const uint8_t *const (&rec)[NT],
                                          double (&acc)[NT]) {
    const int lane = threadIdx.x & 31;
    const int nb = K / COLI_QBLK;
#pragma unroll
    for (int i = 0; i < NT; ++i) acc[i] = 0.0;
#pragma unroll 2
    for (int v = v_lo + lane; v < v_hi; v += 32) {
        const uint4 wv = wrow[v];
#pragma unroll
        for (int i = 0; i < NT; ++i) {
            int s0, s1;
            vec_dot<BITS>(wv, reinterpret_cast<const uint4 *>(rec[i]) + v, V, s0, s1);
            acc[i] = vec_promote<BITS>(v, s0, s1, reinterpret_cast<const int *>(rec[i] + K),
                                       reinterpret_cast<const float *>(rec[i] + K + 4 * nb), acc[i]);
        }
    }
}

// Gate/up stage geometry.  A stage holds R consecutive rows of one matrix;
// each row is split into `slices` vector ranges; the R * slices units are
// spread over the consumer warps, U per warp: warp w takes slice w % slices
// of rows w / slices + k * (PIPE_CONSUMERS / slices), k < U.  When a row has
// V = 96 * slices vectors with slices in {1, 2, 4} (hidden 6144 in every
// format: int2 1, int4 2, int8 4) every lane owns exactly 3 vectors of its
// slice (the register-resident single-token path: 16 units per 24 KB stage,
// U = 2).
struct GuGeom {
    int R, slices, U;
    bool fast;
};
__host__ __device__ inline GuGeom gu_geometry(int H, int bits) {
    const int V = H * bits / 128, RB = H * bits / 8;
    GuGeom g;
    if (V % 96 == 0 && (V / 96 == 1 || V / 96 == 2 || V / 96 == 4)) {
        g.slices = V / 96;
        g.R = 16 / g.slices;
        g.U = 16 / PIPE_CONSUMERS;
        g.fast = true;
    } else {
        g.R = pipe_rows_per_stage(RB);
        g.slices = g.R >= PIPE_CONSUMERS ? 1 : PIPE_CONSUMERS / g.R;
        g.U = g.R * g.slices / PIPE_CONSUMERS;
        g.fast = false;
    }
    return g;
}

// Activation of one token for the vectors a lane owns (VPL of them, lane +
// 32 j past `vbase`), held in registers: codes, the block scales as fp64 and
// the unsigned-offset correction  -off * sum_b xs_b * d_b  of those blocks.
template <int BITS, int VPL> struct LaneAct {
    static constexpr int PL = Fmt<BITS>::PLANES;
    static constexpr int NBV = BITS == 2 ? 2 : 1;  // scales per vector
    uint4 a[VPL][PL];
    double d[VPL][NBV];
    double corr;
    __device__ __forceinline__ void load(const uint8_t *rec, int K, int V, int vbase) {
        const int lane = threadIdx.x & 31;
        const int nb = K / COLI_QBLK;
        const int *xs = reinterpret_cast<const int *>(rec + K);
        const float *xd = reinterpret_cast<const float *>(rec + K + 4 * nb);
        corr = 0.0;
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
            const int v = vbase + lane + 32 * j;
#pragma unroll
            for (int p = 0; p < PL; ++p) a[j][p] = reinterpret_cast<const uint4 *>(rec)[p * V + v];
            if (BITS == 8) {
                d[j][0] = (double)xd[v >> 1];
            } else if (BITS == 4) {
                d[j][0] = (double)xd[v];
                corr = fma(-8.0 * (double)xs[v], d[j][0], corr);
            } else {
                d[j][0] = (double)xd[2 * v];
                d[j][1] = (double)xd[2 * v + 1];
                corr = fma(-2.0 * (double)xs[2 * v], d[j][0], corr);
                corr = fma(-2.0 * (double)xs[2 * v + 1], d[j][1], corr);
            }
        }
    }
    // lane partial of one weight row (its VPL vectors at wrow[vbase + lane + 32 j])
    __device__ __forceinline__ double dot(const uint4 *wrow, int vbase) const {
        const int lane = threadIdx.x & 31;
        const uint32_t base = smem_u32(wrow + vbase + lane);
        double acc = corr;
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
            const uint4 w = lds128(base + 512u * j);
            if (BITS == 8) {
                acc = fma((double)dot_byte(w, a[j][0]), d[j][0], acc);
            } else if (BITS == 4) {
                acc = fma((double)dot_nib(w, a[j][0], a[j][1]), d[j][0], acc);
            } else {
                acc = fma((double)dot_crumb2(w.x, w.y, a[j][0], a[j][1]), d[j][0], acc);
                acc = fma((double)dot_crumb2(w.z, w.w, a[j][2], a[j][3]), d[j][1], acc);
            }
        }
        return acc;
    }
};

// Gate/up consumer work for one stage: row slices assigned to this warp,
// NT tokens; writes the reduced sums to part[row][slice][token].
template <int BITS, int NT>
__device__ __forceinline__ void gateup_stage(const uint8_t *stage, int RB, int V, int H,
                                             const GuGeom g, int row_base, const uint8_t *acts,
                                             int rbH, const int *tok, int i0, double *part_mat,
                                             int ntok) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint8_t *rec[NT];
#pragma unroll
    for (int i = 0; i < NT; ++i) rec[i] = acts + (size_t)tok[i] * rbH;
    const int sl = warp % g.slices;
    const int v_lo = (int)((long long)sl * V / g.slices);
    const int v_hi = (int)((long long)(sl + 1) * V / g.slices);
    for (int k = 0; k < g.U; ++k) {
        const int row = warp / g.slices + k * (PIPE_CONSUMERS / g.slices);
        double acc[NT];
        slice_dot<BITS, NT>(reinterpret_cast<const uint4 *>(stage + (size_t)row * RB), v_lo, v_hi, V,
                            H, rec, acc);
#pragma unroll
        for (int i = 0; i < NT; ++i) {
            const double tot = warp_sum(acc[i]);
            if (lane == 0) part_mat[((row_base + row) * g.slices + sl) * ntok + i0 + i] = tot;
        }
    }
}

// Single-token fast path of one stage (geometry fast: U = 2 rows per warp,
// 3 vectors per lane per row); activations already in registers.
// Per-warp constants of the fast path: slice sl of rows r0 and r0 + rstep.
struct FastGeo {
    int sl, vbase, r0, rstep, slices;
    __device__ __forceinline__ FastGeo(const GuGeom &g, int V) {
        const int warp = threadIdx.x >> 5;
        slices = g.slices;
        sl = warp % g.slices;
        vbase = sl * (V / g.slices);
        rstep = PIPE_CONSUMERS / g.slices;
        r0 = warp / g.slices;
    }
};

// Ring position: slot and phase parity advance together (no divisions).
struct RingPos {
    int slot = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ void next(int ns) {
        if (++slot == ns) {
            slot = 0;
            phase ^= 1u;
        }
    }
};

// The ring as the consumers see it.  A down stage may span two adjacent
// slots (one bulk copy of up to twice the slot size, starting on an even
// slot); the second slot's full phase completes without data.
struct RingView {
    const uint8_t *ring;
    PipeBars *bars;
    int ns;
    int *err;
    volatile int *abort;
    int span = 1;
    long long lim = WAIT_LIMIT_CYCLES;  // limit of the stage waits
};

// Consumer side of releasing one (possibly two-slot) stage: every lane has
// finished reading it.
__device__ __forceinline__ void release_stage(PipeBars *bars, RingPos &rp, int ns, int span) {
    const int lane = threadIdx.x & 31;
    __syncwarp();
    for (int z = 0; z < span; ++z) {
        if (lane == 0) mbar_arrive(&bars->empty[rp.slot]);
        rp.next(ns);
    }
}

// Consumer side of one whole gate/up item on the fast geometry (SL slices of
// the row, R = 16 / SL rows a stage, 2 SL stages a matrix): a warp keeps the
// lane partials of its two rows of every stage in registers and reduces them
// across the lanes once a matrix, so a stage costs its loads and dots only.
// False (abort flag set) if a stage wait ran out.
template <int BITS, int SL>
__device__ __forceinline__ bool gateup_item_fast(const RingView &rv, RingPos &rp, int RB,
                                                 const FastGeo &f, const LaneAct<BITS, 3> &act,
                                                 double *pbuf, size_t part_mat, int ntok) {
    constexpr int R = 16 / SL, SPM = 32 / R, U = 2 * SPM;
    constexpr int SHIFT = U == 4 ? 3 : (U == 8 ? 2 : 1);
    const int lane = threadIdx.x & 31;
#pragma unroll 1
    for (int m = 0; m < 2; ++m) {
        double acc[U];
#pragma unroll
        for (int st = 0; st < SPM; ++st) {
            if (!mbar_wait(&rv.bars->full[rp.slot], rp.phase, rv.err, rv.lim)) {
                *rv.abort = 1;
                return false;
            }
            const uint8_t *stage = rv.ring + (size_t)rp.slot * PIPE_STAGE_MAX;
#pragma unroll
            for (int k = 0; k < 2; ++k)
                acc[2 * st + k] =
                    act.dot(reinterpret_cast<const uint4 *>(stage + (size_t)(f.r0 + k * f.rstep) * RB), f.vbase);
            __syncwarp();
            if (lane == 0) mbar_arrive(&rv.bars->empty[rp.slot]);
            rp.next(rv.ns);
        }
        const double tot = warp_sum_rows<U>(acc);
        if ((lane & ((1 << SHIFT) - 1)) == 0) {
            const int i = lane >> SHIFT, st = i >> 1, k = i & 1;
            const int row = st * R + f.r0 + k * f.rstep;
            pbuf[(size_t)m * part_mat + ((size_t)row * SL + f.sl) * ntok] = tot;
        }
    }
    return true;
}

// 16-byte asynchronous global -> shared copies (L2 only), completed by
// cp_async_wait_all.
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ unsigned ld_relaxed_u32(const unsigned *p) {
    unsigned v;
    asm volatile("ld.relaxed.gpu.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Barrier across every CTA of a cooperative grid; called by one thread per
// CTA between two CTA-level barriers.  `count` is a 64-bit arrival counter
// that only grows: an arrival that returns v belongs to the generation ending
// at (v / nblocks + 1) * nblocks, and the barrier opens when the counter gets
// there (one atomic and, usually, one acquire load per CTA; no reset).
// Bounded: false (and COLI_ETIMEOUT in *err) if the others did not arrive
// within WAIT_LIMIT_CYCLES.
__device__ inline bool grid_barrier(unsigned long long *count, unsigned nblocks, int *err,
                                    long long lim) {
    unsigned long long v;
    asm volatile("atom.add.acq_rel.gpu.u64 %0, [%1], 1;" : "=l"(v) : "l"(count) : "memory");
    const unsigned long long target = (v / nblocks + 1) * nblocks;
    const long long t0 = clock64();
    for (;;) {
        unsigned long long now;
        asm volatile("ld.acquire.gpu.u64 %0, [%1];" : "=l"(now) : "l"(count) : "memory");
        if (now >= target) return true;
        if (clock64() - t0 > lim) {
            atomicExch(err, ERR_TIMEOUT);
            return false;
        }
    }
}

// Down consumer work for one stage: rows w, w + 8, ... of the stage, NT tokens
// starting at pair p; writes e = (float)(sum * row scale) to ebuf.
template <int BITS, int NT>
__device__ __forceinline__ void down_stage(const uint8_t *stage, int RB, int V, int I, int nr,
                                           const float *scales, const uint8_t *recs, int rbI,
                                           int p, float *ebuf, int rows_cap, int row_off) {
    // records of the NT tokens at recs + i rbI; their outputs at pairs p + i
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint8_t *rec[NT];
#pragma unroll
    for (int i = 0; i < NT; ++i) rec[i] = recs + (size_t)i * rbI;
    for (int row = warp; row < nr; row += PIPE_CONSUMERS) {
        const float sc = scales[row];
        double acc[NT];
        slice_dot<BITS, NT>(reinterpret_cast<const uint4 *>(stage + (size_t)row * RB), 0, V, V, I,
                            rec, acc);
#pragma unroll
        for (int i = 0; i < NT; ++i) {
            const double tot = warp_sum(acc[i]);
            if (lane == 0) ebuf[(size_t)(p + i) * rows_cap + row_off + row] = (float)(tot * (double)sc);
        }
    }
}

// Down fast path for one pair: warp w takes rows w + 8 i (i < RPW) of the
// stage, the pair's activation in registers (VPL vectors per lane, full
// rows), and reduces its RPW lane partials across the lanes at once.  RPW is
// the stage's rows per warp rounded up, so no dot is issued for a row the
// stage does not have (except in a shorter last stage).
template <int BITS, int VPL, int RPW>
__device__ __forceinline__ void down_stage_fast(const uint8_t *stage, int RB, int nr,
                                                const float *scales /* shared */,
                                                const LaneAct<BITS, VPL> &act, int p, float *ebuf,
                                                int rows_cap, int row_off) {
    constexpr int U = RPW <= 1 ? 1 : (RPW <= 2 ? 2 : (RPW <= 4 ? 4 : 8));
    constexpr int SHIFT = U == 1 ? 5 : (U == 2 ? 4 : (U == 4 ? 3 : 2));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    double acc[U];
#pragma unroll
    for (int i = 0; i < U; ++i) {
        const int row = warp + PIPE_CONSUMERS * i;
        acc[i] = (i < RPW && row < nr) ? act.dot(reinterpret_cast<const uint4 *>(stage + (size_t)row * RB), 0)
                                       : 0.0;
    }
    const double tot = warp_sum_rows<U>(acc);
    const int i = lane >> SHIFT;
    const int row = warp + PIPE_CONSUMERS * i;
    if ((lane & ((1 << SHIFT) - 1)) == 0 && i < RPW && row < nr)
        ebuf[(size_t)p * rows_cap + row_off + row] = (float)(tot * (double)scales[row]);
}

// Down rows of one single-token expert over its SUBS stages (stage sb holds
// rows sb * down_rows + [0, nr)), warp w taking rows w + 8 i (i < RPW) of
// each: the lane partials of all SUBS * RPW rows stay in registers and are
// reduced across the lanes once, after the expert's last stage, instead of
// once a stage.  Requires down_rows == 8 * RPW (every stage but the last
// full).  False (abort flag set) if a stage wait ran out.
template <int BITS, int VPL, int RPW, int SUBS>
__device__ __forceinline__ bool down_expert_deferred(const RingView &rv, RingPos &rp, int RB, int nrows,
                                                     const float *scales /* shared, this expert */,
                                                     const LaneAct<BITS, VPL> &act, int p, float *ebuf,
                                                     int rows_cap) {
    constexpr int N = RPW * SUBS;
    static_assert(N <= 16, "at most 16 deferred rows per warp");
    constexpr int U = N <= 4 ? 4 : (N <= 8 ? 8 : 16);
    constexpr int SHIFT = U == 4 ? 3 : (U == 8 ? 2 : 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    double acc[U];
#pragma unroll
    for (int i = N; i < U; ++i) acc[i] = 0.0;
#pragma unroll
    for (int sb = 0; sb < SUBS; ++sb) {
        if (!mbar_wait(&rv.bars->full[rp.slot], rp.phase, rv.err, rv.lim)) {
            *rv.abort = 1;
            return false;
        }
        const uint8_t *stage = rv.ring + (size_t)rp.slot * PIPE_STAGE_MAX;
        const int nr = min(8 * RPW, nrows - sb * 8 * RPW);
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
            const int row = warp + PIPE_CONSUMERS * i;
            acc[sb * RPW + i] =
                row < nr ? act.dot(reinterpret_cast<const uint4 *>(stage + (size_t)row * RB), 0) : 0.0;
        }
        release_stage(rv.bars, rp, rv.ns, rv.span);
    }
    const double tot = warp_sum_rows<U>(acc);
    const int j = lane >> SHIFT, sb = j / RPW, i = j - sb * RPW;
    const int row = sb * 8 * RPW + warp + PIPE_CONSUMERS * i;
    if ((lane & ((1 << SHIFT) - 1)) == 0 && j < N && row < nrows)
        ebuf[(size_t)p * rows_cap + row] = (float)(tot * (double)scales[row]);
    return true;
}

template <int BITS, int VPL>
__device__ __forceinline__ void down_stage_fast_any(int rpw, const uint8_t *stage, int RB, int nr,
                                                    const float *scales, const LaneAct<BITS, VPL> &act,
                                                    int p, float *ebuf, int rows_cap, int row_off) {
    switch (rpw) {
        case 1: down_stage_fast<BITS, VPL, 1>(stage, RB, nr, scales, act, p, ebuf, rows_cap, row_off); break;
        case 2: down_stage_fast<BITS, VPL, 2>(stage, RB, nr, scales, act, p, ebuf, rows_cap, row_off); break;
        case 3: down_stage_fast<BITS, VPL, 3>(stage, RB, nr, scales, act, p, ebuf, rows_cap, row_off); break;
        case 4: down_stage_fast<BITS, VPL, 4>(stage, RB, nr, scales, act, p, ebuf, rows_cap, row_off); break;
        default: down_stage_fast<BITS, VPL, 8>(stage, RB, nr, scales, act, p, ebuf, rows_cap, row_off); break;
    }
}

// ===========================================================================
// The whole layer for few tokens in one persistent cooperative launch (one
// CTA per SM, all co-resident).  One ring of weight stages runs through the
// kernel: the shared experts' gate/up rows (issued while routing is still in
// progress: they need none), the routed experts' gate/up rows, then the down
// rows of this CTA's output-row range for every active expert (they need no
// h, so they stream while the gate/up items finish elsewhere).
//   P1  fp64 logits of experts b, b + grid, ...; Q8_0(x) records of a share
//       of the blocks, to global memory.            -- grid barrier --
//   P2  every CTA copies the records, selects every token's experts and
//       builds the batch-union tables in shared memory (CTA 0 publishes them).
//   P3  gate/up items + SwiGLU + Q8_0(h) records, to global memory; each item
//       adds one to its expert's count.
//   P4  experts in the down order (shared first): once an expert's count is
//       complete, the h-fetch warp copies its h records into one of the nh
//       shared slots and the consumers run its down rows; then the fp64
//       combine of this CTA's rows, shared experts first.
struct DecodeArgs {
    const float *x;
    const float *Wr;
    const float *bias;
    int T, H, I, E, S, G, gk, k;
    float rsf;
    float top_p;        // adaptive expert top-p (0 or >= 1: off)
    RouteWs ws;
    const ExpertDev *experts;
    uint8_t *xrec;
    int8_t *xq;
    float *xd;
    uint8_t *hrec;
    int8_t *hq;
    float *hd;
    float *out;
    double *out_partial;        // if set: the unrounded fp64 sum of this handle's slots instead of out
    int *err;
    unsigned long long *gbar;   // grid-barrier arrival counter
    int *hcnt;                  // per active expert: gate/up items whose h records are written
    int ns, pmax;
    int rows_cap;       // output rows per CTA (max) in P4
    int down_rows;      // down rows per stage
    int down_span;      // ring slots per down stage (1, or 2: one copy across two adjacent slots)
    int nh;             // shared slots for the h records of active experts (<= DECODE_MAX_HSLOTS)
    int h_alias;        // 1: the slots reuse the x records' space, so they fill only after P3
    int ptr_smem;       // 1: every expert's code pointers are staged in shared memory in P1
    const long long *wait_limit;  // SM cycles a wait on progress may last (drains keep the default)
};

constexpr int DECODE_MAX_HSLOTS = 16;
// every expert's gate/up/down code pointers and down scales pointer staged in
// shared memory while routing runs, when E + S is at most this
constexpr int DECODE_PTR_SMEM_MAX = 320;

struct DecodeSmem {
    size_t select, idxw, cnt, red, tables, act, hslot, hbar, eptrs, ebuf, part, dscale, eptr, ring,
        total;
};

__host__ __device__ inline DecodeSmem decode_smem(int T, int H, int I, int E, int S, int G, int k,
                                                  int pmax, int slices, int rows_cap, int ns,
                                                  int nh, int h_alias, int ptr_smem) {
    DecodeSmem d;
    size_t o = pipe_hdr_bytes();
    d.ring = o;
    o += (size_t)ns * PIPE_STAGE_MAX;
    d.select = o;
    o += align128(select_smem_bytes(E, G));
    d.idxw = o;
    o += align128((size_t)T * k * 8);
    d.cnt = o;
    o += align128((size_t)E * 4);
    d.red = o;
    o += align128((size_t)2 * 8 * PIPE_MAX_TOK * 8);
    d.tables = o;
    o += align128((size_t)(3 * (E + S) + 1 + 3 * pmax + 4) * 4);
    const size_t xa = (size_t)T * rec_bytes(H), ha = (size_t)nh * T * rec_bytes(I);
    d.act = o;                            // Q8_0(x) records of the T tokens
    if (h_alias) {                        // nh slots of T h records each, in the same space
        d.hslot = o;
        o += align128(xa > ha ? xa : ha);
    } else {
        o += align128(xa);
        d.hslot = o;
        o += align128(ha);
    }
    d.hbar = o;                           // h_full[nh], h_empty[nh], x_free
    o += align128((size_t)(2 * nh + 1) * 8);
    d.eptrs = o;                          // 4 pointers per expert (ptr_smem only)
    o += ptr_smem ? align128((size_t)(E + S) * 4 * sizeof(void *)) : 0;
    d.ebuf = o;
    o += align128((size_t)pmax * rows_cap * 4);
    d.part = o;
    const int ntok = T < PIPE_MAX_TOK ? T : PIPE_MAX_TOK;
    o += align128((size_t)2 * 2 * 32 * slices * ntok * 8);
    d.dscale = o;                         // down-row scales of this CTA, per active expert
    const int amax = (E < T * k ? E : T * k) + S;
    o += align128((size_t)amax * (rows_cap + 4) * 4);
    d.eptr = o;                           // gate, up, down code pointers per active expert
    o += align128((size_t)amax * 3 * sizeof(void *));
    d.total = o;
    return d;
}


// One decision for all 8 consumer warps: whether the launch was aborted.
// Every consumer warp calls it at the same point; one thread reads the flag
// between two consumer barriers, so no warp leaves while another waits at a
// later barrier for it.
__device__ __forceinline__ bool consumers_aborted(volatile int *abort, int *flag_smem) {
    named_bar(1, 256);
    if (threadIdx.x == 0) *(volatile int *)flag_smem = *abort;
    named_bar(1, 256);
    return *(volatile int *)flag_smem != 0;
}

// P4 of the decode kernel: the consumer side of the down stages of this CTA's
// output rows, one active expert after another.  VPL = vectors per lane of
// the h activation (1, 2, 4: register-resident activation, loaded once per
// single-token expert before its first stage wait); VPL = 0 is the generic
// shared-memory path for any other width.
struct EpiBars {
    uint64_t part_full[2];   // the 8 consumer warps finished an item's partials
    uint64_t part_free[2];   // the epilogue warp finished reading them
};

struct DownLoop {
    const int *off;
    int n_active, S, T, subs, ns, down_rows, rows_cap, r0, nrows, RBI, VI, I, rbI, span;
    long long lim;
    const uint8_t *ring;
    const float *dscale;
    const uint8_t *hslots;   // nh slots of T h records each, filled by the epilogue warp
    int nh;
    uint64_t *hfull;         // [nh] an expert's h records are in its slot (32 cp.async arrivals)
    uint64_t *hempty;        // [nh] the 8 consumer warps are done with that slot
    float *ebuf;
    PipeBars *bars;
    volatile int *abort;
    int *err;
};

// Order of the down phase: the shared experts first (their h is complete
// earliest: their gate/up items come first), then the routed ones.
__device__ __forceinline__ int down_slot(int q, int n_active, int S) {
    return q < S ? n_active - S + q : q - S;
}

template <int BITS, int VPL, int MAXT>
__device__ __forceinline__ bool down_loop(const DownLoop &d, RingPos &rp) {
    const int lane = threadIdx.x & 31;
    const int rpw = (d.down_rows + PIPE_CONSUMERS - 1) / PIPE_CONSUMERS;
    for (int q = 0; q < d.n_active; ++q) {
        const int a = down_slot(q, d.n_active, d.S);
        const int p0 = d.off[a], ne = d.off[a + 1] - p0;
        // this expert's h records: slot q % nh, filled once all its gate/up
        // items (any CTA's) are written
        const int hs = q % d.nh;
        const uint8_t *recs = d.hslots + (size_t)hs * d.T * d.rbI;
        if (!mbar_wait(&d.hfull[hs], (uint32_t)((q / d.nh) & 1), d.err, d.lim)) {
            *d.abort = 1;
            return false;
        }
        bool expert_ok = true;
        LaneAct<BITS, (VPL > 0 ? VPL : 1)> act;
        int done = -1;
        if constexpr (VPL > 0) {
            if (MAXT == 1 || ne == 1) {
                act.load(recs, d.I, d.VI, 0);
                // whole expert at once where the stage geometry allows
                const float *sc_a = d.dscale + a * (d.rows_cap + 4);
                const RingView rv{d.ring, d.bars, d.ns, d.err, d.abort, d.span, d.lim};
                if (d.down_rows == 8 * rpw) {
#define COLI_DEFER(R, SB) done = down_expert_deferred<BITS, VPL, R, SB>(rv, rp, d.RBI, d.nrows, sc_a, act, p0, d.ebuf, d.rows_cap)
                    if (rpw == 6 && d.subs == 1) COLI_DEFER(6, 1);
                    else if (rpw == 6 && d.subs == 2) COLI_DEFER(6, 2);
                    else if (rpw == 4 && d.subs == 1) COLI_DEFER(4, 1);
                    else if (rpw == 2 && d.subs == 1) COLI_DEFER(2, 1);
                    else if (rpw == 3 && d.subs == 1) COLI_DEFER(3, 1);
                    else if (rpw == 3 && d.subs == 2) COLI_DEFER(3, 2);
                    else if (rpw == 3 && d.subs == 3) COLI_DEFER(3, 3);
                    else if (rpw == 3 && d.subs == 4) COLI_DEFER(3, 4);
                    else if (rpw == 4 && d.subs == 2) COLI_DEFER(4, 2);
                    else if (rpw == 2 && d.subs == 2) COLI_DEFER(2, 2);
                    else if (rpw == 2 && d.subs == 3) COLI_DEFER(2, 3);
                    else if (rpw == 2 && d.subs == 4) COLI_DEFER(2, 4);
#undef COLI_DEFER
                }
                if (done == 0) return false;
            }
        }
        for (int sb = 0; done != 1 && sb < d.subs; ++sb) {
            if (!mbar_wait(&d.bars->full[rp.slot], rp.phase, d.err, d.lim)) {
                *d.abort = 1;
                expert_ok = false;
                break;
            }
            const int rs = d.r0 + sb * d.down_rows;
            const int nr = min(d.down_rows, d.r0 + d.nrows - rs);
            const uint8_t *stage = d.ring + (size_t)rp.slot * PIPE_STAGE_MAX;
            const int ro = rs - d.r0;
            const float *sc = d.dscale + a * (d.rows_cap + 4) + ro;
            if constexpr (VPL > 0) {
                if (MAXT == 1 || ne == 1) {
                    down_stage_fast_any<BITS, VPL>(rpw, stage, d.RBI, nr, sc, act, p0, d.ebuf, d.rows_cap, ro);
                } else {
                    for (int i = 0; i < ne; ++i) {
                        LaneAct<BITS, VPL> ta;
                        ta.load(recs + (size_t)i * d.rbI, d.I, d.VI, 0);
                        down_stage_fast_any<BITS, VPL>(rpw, stage, d.RBI, nr, sc, ta, p0 + i, d.ebuf,
                                                       d.rows_cap, ro);
                    }
                }
            } else if constexpr (MAXT == 1) {
                down_stage<BITS, 1>(stage, d.RBI, d.VI, d.I, nr, sc, recs, d.rbI, p0, d.ebuf, d.rows_cap, ro);
            } else {
                for (int i0 = 0; i0 < ne; i0 += PIPE_PASS_TOK) {
                    const int nn = min(PIPE_PASS_TOK, ne - i0);
                    const uint8_t *r = recs + (size_t)i0 * d.rbI;
                    switch (nn) {
                        case 1: down_stage<BITS, 1>(stage, d.RBI, d.VI, d.I, nr, sc, r, d.rbI, p0 + i0, d.ebuf, d.rows_cap, ro); break;
                        case 2: down_stage<BITS, 2>(stage, d.RBI, d.VI, d.I, nr, sc, r, d.rbI, p0 + i0, d.ebuf, d.rows_cap, ro); break;
                        case 3: down_stage<BITS, 3>(stage, d.RBI, d.VI, d.I, nr, sc, r, d.rbI, p0 + i0, d.ebuf, d.rows_cap, ro); break;
                        default: down_stage<BITS, 4>(stage, d.RBI, d.VI, d.I, nr, sc, r, d.rbI, p0 + i0, d.ebuf, d.rows_cap, ro); break;
                    }
                }
            }
            release_stage(d.bars, rp, d.ns, d.span);
        }
        if (!expert_ok) return false;
        // the slot may be refilled
        __syncwarp();
        if (lane == 0) mbar_arrive(&d.hempty[hs]);
    }
    return true;
}

// Stage cursor of one CTA: its gate/up items (j-th item, matrix step m), then
// its down stages (active expert a, row sub-range sb).
struct StageCursor {
    int j = 0, m = 0, a = 0, sb = 0;
    bool down = false;
    __device__ __forceinline__ void next(int my_items, int steps, int subs) {
        if (!down) {
            if (++m == steps) {
                m = 0;
                if (++j >= my_items) {
                    down = true;
                    a = 0;
                    sb = 0;
                }
            }
        } else if (++sb == subs) {
            sb = 0;
            ++a;
        }
    }
};

// MAXT: the most tokens the instance handles (1, or PIPE_MAX_TOK); the
// single-token instance carries none of the multi-token code, which keeps the
// hot loops of every phase compact in the instruction caches.
template <int BITS, int MAXT>
__global__ void __launch_bounds__(DECODE_THREADS, 1) k_moe_decode(DecodeArgs fa) {
    extern __shared__ __align__(128) uint8_t smem[];
    PipeBars *bars = reinterpret_cast<PipeBars *>(smem);
    EpiBars *ebars = reinterpret_cast<EpiBars *>(smem + sizeof(PipeBars) + 8);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int T = fa.T, H = fa.H, I = fa.I, E = fa.E, S = fa.S, k = fa.k;
    // shared experts in the active list (the slot layout always has S of them)
    const int Sa = fa.ws.shared_active(S);
    const int RB = H * BITS / 8, V = H * BITS / 128;
    const int RBI = I * BITS / 8, VI = I * BITS / 128;
    const GuGeom geo = gu_geometry(H, BITS);
    const int R = geo.R, slices = geo.slices, spm = 32 / R, steps = 2 * spm;
    const int nchunk = I / 32, rbH = rec_bytes(H), rbI = rec_bytes(I), nbH = H / COLI_QBLK;
    const int ns = fa.ns, G = gridDim.x;
    const long long lim = *fa.wait_limit;
    const DecodeSmem L = decode_smem(T, H, I, E, S, fa.G, k, fa.pmax, slices, fa.rows_cap, ns,
                                     fa.nh, fa.h_alias, fa.ptr_smem);
    uint8_t *ring = smem + L.ring;
    SelectSmem sm = carve_select(smem + L.select, E, fa.G);
    int *idx_s = reinterpret_cast<int *>(smem + L.idxw);
    float *w_s = reinterpret_cast<float *>(idx_s + T * k);
    int *cnt = reinterpret_cast<int *>(smem + L.cnt);
    double *red = reinterpret_cast<double *>(smem + L.red);
    RouteWs lw = fa.ws;
    lw.active = reinterpret_cast<int32_t *>(smem + L.tables);
    lw.off = lw.active + (E + S);
    lw.act_of = lw.off + (E + S + 1);
    lw.pair_tok = lw.act_of + (E + S);
    lw.pair_slot = lw.pair_tok + fa.pmax;
    lw.tok_pair = lw.pair_slot + fa.pmax;
    lw.n_active = lw.tok_pair + fa.pmax;
    int *flags = lw.n_active + 1;
    uint8_t *acts = smem + L.act;       // x records (P2, P3)
    uint8_t *hslots = smem + L.hslot;   // h records of active experts (P3, P4)
    uint64_t *hfull = reinterpret_cast<uint64_t *>(smem + L.hbar);
    uint64_t *hempty = hfull + fa.nh;
    uint64_t *xfree = hempty + fa.nh;   // the consumers are done with the x records (after P3)
    // gate, up, down code pointers and the down scales pointer of every expert
    // (ptr_smem), staged by the epilogue warp while routing runs
    const void **eptrs = reinterpret_cast<const void **>(smem + L.eptrs);
    float *ebuf = reinterpret_cast<float *>(smem + L.ebuf);
    double *part = reinterpret_cast<double *>(smem + L.part);
    float *dscale = reinterpret_cast<float *>(smem + L.dscale);   // [active][rows_cap + 4]
    const int ntok = T < PIPE_MAX_TOK ? T : PIPE_MAX_TOK;
    const size_t part_mat = (size_t)32 * slices * ntok;
    const int rbase = H / G, rrem = H % G;
    const int r0 = blockIdx.x * rbase + min((int)blockIdx.x, rrem);
    const int nrows = rbase + ((int)blockIdx.x < rrem ? 1 : 0);
    const int subs = (nrows + fa.down_rows - 1) / fa.down_rows;
    const size_t gu_bytes = (size_t)R * RB;
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ebars->part_full[i], PIPE_CONSUMERS);
            mbar_init(&ebars->part_free[i], 1);
        }
        for (int i = 0; i < fa.nh; ++i) {
            mbar_init(&hfull[i], 32);   // one cp.async completion arrival per epilogue lane
            mbar_init(&hempty[i], PIPE_CONSUMERS);
        }
        mbar_init(xfree, PIPE_CONSUMERS);
    }
    pipe_init(bars, ns);
    __syncthreads();
    volatile int *abort = &bars->abort;
    const int n_shared_items = Sa * nchunk;
    auto item_of = [&](int j) { return (int)blockIdx.x + j * G; };
    auto item_expert_chunk = [&](int item, int n_active, int &a, int &e, int &c) {
        if (item < n_shared_items) {
            const int q = item / nchunk;
            a = n_active - Sa + q;
            e = E + q;
            c = item - q * nchunk;
        } else {
            const int q = (item - n_shared_items) / nchunk;
            a = q;
            e = -1;  // looked up in the tables by the caller
            c = item - n_shared_items - q * nchunk;
        }
    };

    if (warp == PIPE_CONSUMERS) {
        // ------------------------------ producer (lane 0 issues)
        StageCursor cur;
        RingPos rp;
        const uint64_t pol = l2_evict_first_policy();
        int issued = 0;
        // routing goes first: the consumers release this barrier once the
        // selection's scores are in shared memory, so neither the router
        // weights nor the grid barrier nor those loads queue behind the
        // shared expert's bulk copies in the memory system
        asm volatile("bar.sync 4, %0;" ::"r"(32 * (PIPE_CONSUMERS + 1)) : "memory");
        int q_ld = -1;
        const uint8_t *sh_gate = nullptr, *sh_up = nullptr;
        while (lane == 0 && issued < ns && item_of(cur.j) < n_shared_items) {
            const int item = item_of(cur.j);
            const int q = item / nchunk;
            if (q != q_ld) {
                sh_gate = fa.experts[E + q].gate.codes;
                sh_up = fa.experts[E + q].up.codes;
                q_ld = q;
            }
            const int row0 = (item - q * nchunk) * 32 + (cur.m % spm) * R;
            mbar_expect_tx(&bars->full[rp.slot], (uint32_t)gu_bytes);
            bulk_g2s_hint(ring + (size_t)rp.slot * PIPE_STAGE_MAX, (cur.m < spm ? sh_gate : sh_up) + (size_t)row0 * RB,
                          (uint32_t)gu_bytes, &bars->full[rp.slot], pol);
            ++issued;
            rp.next(ns);
            cur.next(1 << 30, steps, subs);
        }
        if (lane == 0) {
            // the rest of this CTA's shared gate/up stages (beyond the ring)
            // into L2, then the shared experts' down rows of this CTA
            StageCursor c2 = cur;
            for (int n = 0; n < steps && item_of(c2.j) < n_shared_items; ++n) {
                const int item = item_of(c2.j);
                const int q = item / nchunk;
                const ExpertDev &ex = fa.experts[E + q];
                const int row0 = (item - q * nchunk) * 32 + (c2.m % spm) * R;
                bulk_prefetch_l2((c2.m < spm ? ex.gate.codes : ex.up.codes) + (size_t)row0 * RB, (uint32_t)gu_bytes);
                c2.next(1 << 30, steps, subs);
            }
            for (int i = 0; i < Sa; ++i)
                bulk_prefetch_l2(fa.experts[E + i].down.codes + (size_t)r0 * RBI, (uint32_t)(nrows * RBI));
        }
        __syncwarp();
        named_bar(2, DECODE_THREADS);        // routing tables ready (or aborted)
        if (*abort) {
            if (lane == 0) pipe_drain(bars, ns, issued, 0, fa.err);
            return;
        }
        const int n_active = *lw.n_active;
        // code pointers of every active expert into shared memory, one
        // parallel round of loads, so that issuing a stage reads no global
        // memory
        const uint8_t **ptab = reinterpret_cast<const uint8_t **>(smem + L.eptr);
        for (int a = lane; a < n_active; a += 32) {
            const int e = lw.active[a];
            if (fa.ptr_smem) {
                ptab[3 * a] = static_cast<const uint8_t *>(eptrs[4 * e]);
                ptab[3 * a + 1] = static_cast<const uint8_t *>(eptrs[4 * e + 1]);
                ptab[3 * a + 2] = static_cast<const uint8_t *>(eptrs[4 * e + 2]);
            } else {
                const ExpertDev ex = fa.experts[e];
                ptab[3 * a] = ex.gate.codes;
                ptab[3 * a + 1] = ex.up.codes;
                ptab[3 * a + 2] = ex.down.codes;
            }
        }
        __syncwarp();
        if (lane != 0) return;
        const int n_items = n_active * nchunk;
        const int my_items = n_items > (int)blockIdx.x ? (n_items - 1 - (int)blockIdx.x) / G + 1 : 0;
        const int n_total = my_items * steps + n_active * subs;
        if (cur.j >= my_items && !cur.down) {  // no gate/up work was pending
            cur.down = true;
            cur.a = 0;
            cur.sb = 0;
        }
        auto desc = [&](const StageCursor &c, uint32_t &bytes) -> const uint8_t * {
            if (!c.down) {
                int a, e, ch;
                item_expert_chunk(item_of(c.j), n_active, a, e, ch);
                const int up = c.m < spm ? 0 : 1;
                bytes = (uint32_t)gu_bytes;
                return ptab[3 * a + up] + (size_t)(ch * 32 + (c.m - up * spm) * R) * RB;
            }
            const int rs = r0 + c.sb * fa.down_rows;
            const int nr = min(fa.down_rows, r0 + nrows - rs);
            bytes = (uint32_t)(nr * RBI);
            return ptab[3 * down_slot(c.a, n_active, Sa) + 2] + (size_t)rs * RBI;
        };
        // No L2 prefetch ahead of the ring: the bulk-copy unit of the SM is
        // what limits the issue rate, and a prefetch costs it as much as the
        // copy itself; ns stages in flight already cover the DRAM latency.
        long long si = issued;  // ring slots filled so far
        for (int st = issued; st < n_total; ++st) {
            // a down stage may take two adjacent slots (it starts on an even
            // slot: every gate/up item is an even number of stages and ns is
            // even then); both must be free
            const int span = cur.down ? fa.down_span : 1;
            RingPos wp = rp;
            bool free_ok = true;
            for (int z = 0; z < span && free_ok; ++z) {
                if (si + z >= ns && !mbar_wait_sleepy(&bars->empty[wp.slot], wp.phase ^ 1u, fa.err, lim))
                    free_ok = false;
                wp.next(ns);
            }
            if (!free_ok) {
                pipe_drain(bars, ns, si, si - ns > 0 ? si - ns : 0, fa.err);
                return;
            }
            uint32_t bytes;
            const uint8_t *src = desc(cur, bytes);
            mbar_expect_tx(&bars->full[rp.slot], bytes);
            bulk_g2s_hint(ring + (size_t)rp.slot * PIPE_STAGE_MAX, src, bytes, &bars->full[rp.slot], pol);
            rp.next(ns);
            for (int z = 1; z < span; ++z) {  // the second slot's phase completes with no data
                mbar_arrive(&bars->full[rp.slot]);
                rp.next(ns);
            }
            si += span;
            cur.next(my_items, steps, subs);
        }
        return;  // the consumers wait for every copy
    }

    if (warp == PIPE_CONSUMERS + 2) {
        // ------------------------------ h-fetch warp: the h records of every
        // active expert, in the down order, into the nh shared slots as soon
        // as all its gate/up items (any CTA's) are counted -- many experts'
        // copies in flight at once, and no grid barrier: a CTA starts its
        // down rows of an expert as soon as that expert's h is complete.
        named_bar(2, DECODE_THREADS);
        bool ok = !*abort;
        const int nh = fa.nh;
        if (ok) {
            const int n_active = *lw.n_active;
            // slots in the x records' space: only once every consumer warp is done with them
            if (fa.h_alias && !mbar_wait_sleepy(xfree, 0, fa.err, lim)) ok = false;
            for (int q = 0; ok && q < n_active; ++q) {
                const int a = down_slot(q, n_active, Sa), slot = q % nh;
                if (q >= nh && !mbar_wait_sleepy(&hempty[slot], (uint32_t)((q / nh - 1) & 1), fa.err, lim)) {
                    ok = false;
                    break;
                }
                int ready = 1;
                if (lane == 0) {
                    // relaxed polls with a back-off (no fence per poll), then
                    // one acquire of the complete count
                    const long long t0 = clock64();
                    while ((int)ld_relaxed_u32(reinterpret_cast<const unsigned *>(fa.hcnt + a)) < nchunk) {
                        if (*abort) {
                            ready = 0;
                            break;
                        }
                        if (clock64() - t0 > lim) {
                            atomicExch(fa.err, ERR_TIMEOUT);
                            ready = 0;
                            break;
                        }
                        __nanosleep(200);
                    }
                    if (ready && (int)ld_acquire_u32(reinterpret_cast<const unsigned *>(fa.hcnt + a)) < nchunk)
                        ready = 0;  // unreachable: the count never decreases within a launch
                }
                ready = __shfl_sync(0xffffffffu, ready, 0);
                __syncwarp();  // every lane's reads below come after lane 0's acquire
                if (!ready) {
                    ok = false;
                    break;
                }
                const int p0 = lw.off[a], ne = lw.off[a + 1] - p0;
                const uint8_t *src = fa.hrec + (size_t)p0 * rbI;
                uint8_t *dst = hslots + (size_t)slot * T * rbI;
                for (int i = lane; i < ne * rbI / 16; i += 32) cp_async16(dst + 16 * i, src + 16 * i);
                cp_async_arrive_noinc(&hfull[slot]);  // each lane: once its copies land
            }
        }
        if (!ok) *abort = 1;
        cp_async_wait_all();  // no copy lands in shared memory after this warp leaves
        return;
    }

    if (warp == PIPE_CONSUMERS + 1) {
        // ------------------------------ epilogue warp.  While routing runs:
        // every expert's code pointers into shared memory (ptr_smem).  P3:
        // SwiGLU + Q8_0(h) of every item, off the consumers' critical path;
        // each item's count is released once its h records are written.
        if (fa.ptr_smem) {
            for (int e = lane; e < E + S; e += 32) {
                const ExpertDev &ex = fa.experts[e];
                eptrs[4 * e] = ex.gate.codes;
                eptrs[4 * e + 1] = ex.up.codes;
                eptrs[4 * e + 2] = ex.down.codes;
                eptrs[4 * e + 3] = ex.down.scales;
            }
        }
        named_bar(2, DECODE_THREADS);
        if (*abort) return;
        const int n_active = *lw.n_active;
        const int n_items = n_active * nchunk;
        int n = 0;
        for (int item = blockIdx.x; item < n_items; item += G, ++n) {
            const int buf = n & 1;
            int a, e, c;
            item_expert_chunk(item, n_active, a, e, c);
            if (e < 0) e = lw.active[a];
            const int p0 = lw.off[a];
            const int ne = min(lw.off[a + 1] - p0, PIPE_MAX_TOK);
            const ExpertDev ex = fa.experts[e];
            const float sg = __ldg(ex.gate.scales + c * 32 + lane);
            const float su = __ldg(ex.up.scales + c * 32 + lane);
            if (!mbar_wait_sleepy(&ebars->part_full[buf], (uint32_t)((n >> 1) & 1), fa.err, lim)) {
                *abort = 1;
                break;
            }
            const double *pbuf = part + (size_t)buf * 2 * part_mat;
            for (int i = 0; i < ne; ++i) {
                double ag = 0.0, au = 0.0;
                for (int sl = 0; sl < slices; ++sl) {
                    ag += pbuf[((size_t)lane * slices + sl) * ntok + i];
                    au += pbuf[part_mat + ((size_t)lane * slices + sl) * ntok + i];
                }
                const float g = (float)(ag * (double)sg);
                const float u = (float)(au * (double)su);
                const double gd = (double)g;
                const float h = (float)((gd / (1.0 + exp(-gd))) * (double)u);
                const int pr = p0 + i;
                q8_block_to_record<BITS>(h, c, I, fa.hrec + (size_t)pr * rbI,
                                         fa.hq + (int64_t)pr * I, fa.hd + (int64_t)pr * (I / COLI_QBLK));
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&ebars->part_free[buf]);
                red_release_add(fa.hcnt + a, 1);  // the item's h records before its count
            }
        }
        return;
    }

    // ---------------------------------- consumers
    // P1: logits of experts b, b + G, ... (two per pass, loads issued four
    // iterations at a time) and a share of Q8_0(x).  Every consumer thread
    // first requests its first router-weight lines into L2; the producer's
    // shared-expert bulk copies wait (barrier 4) until the selection's scores
    // are loaded, so the latency-bound routing steps do not queue behind them.
    if ((int)blockIdx.x < E) {
        const int e1 = (int)blockIdx.x + G;
        for (int i = tid; i < H / 4 && i < 4 * 256; i += 256) {
            asm volatile("prefetch.global.L2 [%0];" ::"l"(fa.Wr + (int64_t)blockIdx.x * H + 4 * i));
            if (e1 < E) asm volatile("prefetch.global.L2 [%0];" ::"l"(fa.Wr + (int64_t)e1 * H + 4 * i));
        }
    }
    for (int e0 = blockIdx.x; e0 < E; e0 += 2 * G) {
        const int e1 = e0 + G;
        const bool two = e1 < E;
        double acc[2][MAXT];
#pragma unroll
        for (int t = 0; t < MAXT; ++t) acc[0][t] = acc[1][t] = 0.0;
        const float4 *w40 = reinterpret_cast<const float4 *>(fa.Wr + (int64_t)e0 * H);
        const float4 *w41 = reinterpret_cast<const float4 *>(fa.Wr + (int64_t)(two ? e1 : e0) * H);
        const int H4 = H / 4;
        // all of a thread's router-weight loads in flight at once where the
        // registers allow (hidden 6144: 6 float4 per thread and expert)
        constexpr int LU = MAXT == 1 ? 6 : 4;
        for (int i0 = tid; i0 < H4; i0 += LU * 256) {
            float4 wa[LU], wb[LU];
#pragma unroll
            for (int u = 0; u < LU; ++u) {
                const int i = i0 + u * 256;
                wa[u] = (i < H4) ? __ldg(w40 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
                wb[u] = (i < H4) ? __ldg(w41 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            }

#pragma unroll
            for (int t = 0; t < MAXT; ++t) {
                if (t < T) {
                    float4 xv[LU];
#pragma unroll
                    for (int u = 0; u < LU; ++u) {
                        const int i = i0 + u * 256;
                        xv[u] = (i < H4) ? __ldg(reinterpret_cast<const float4 *>(fa.x + (int64_t)t * H) + i)
                                         : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
#pragma unroll
                    for (int u = 0; u < LU; ++u) {
                        acc[0][t] = fma((double)xv[u].x, (double)wa[u].x, acc[0][t]);
                        acc[0][t] = fma((double)xv[u].y, (double)wa[u].y, acc[0][t]);
                        acc[0][t] = fma((double)xv[u].z, (double)wa[u].z, acc[0][t]);
                        acc[0][t] = fma((double)xv[u].w, (double)wa[u].w, acc[0][t]);
                        acc[1][t] = fma((double)xv[u].x, (double)wb[u].x, acc[1][t]);
                        acc[1][t] = fma((double)xv[u].y, (double)wb[u].y, acc[1][t]);
                        acc[1][t] = fma((double)xv[u].z, (double)wb[u].z, acc[1][t]);
                        acc[1][t] = fma((double)xv[u].w, (double)wb[u].w, acc[1][t]);
                    }
                }
            }
        }
#pragma unroll
        for (int t = 0; t < MAXT; ++t) {
            if (t < T) {
                const double v0 = warp_sum(acc[0][t]);
                const double v1 = warp_sum(acc[1][t]);
                if (lane == 0) {
                    red[(0 * PIPE_CONSUMERS + warp) * PIPE_MAX_TOK + t] = v0;
                    red[(1 * PIPE_CONSUMERS + warp) * PIPE_MAX_TOK + t] = v1;
                }
            }
        }
        named_bar(1, 256);
        if (tid < 2 * T && (tid < T || two)) {
            const int jj = tid / T, t = tid % T;
            const int e = jj ? e1 : e0;
            double l = 0.0;
            for (int w = 0; w < PIPE_CONSUMERS; ++w) l += red[(jj * PIPE_CONSUMERS + w) * PIPE_MAX_TOK + t];
            const double sg = 1.0 / (1.0 + exp(-l));
            fa.ws.s[(int64_t)t * E + e] = sg;
            fa.ws.c[(int64_t)t * E + e] = sg + (double)fa.bias[e];
        }
        named_bar(1, 256);
    }
    if (blockIdx.x == 0)  // this launch's h-record counts start at zero
        for (int i = tid; i < (E < T * k ? E : T * k) + S; i += 256) fa.hcnt[i] = 0;
    for (int blk = blockIdx.x * PIPE_CONSUMERS + warp; blk < T * nbH; blk += G * PIPE_CONSUMERS) {
        const int t = blk / nbH, b = blk % nbH;
        const float v = __ldg(fa.x + (int64_t)t * H + b * COLI_QBLK + lane);
        q8_block_to_record<BITS>(v, b, H, fa.xrec + (size_t)t * rbH, fa.xq + (int64_t)t * H,
                                 fa.xd + (int64_t)t * nbH);
    }
    named_bar(1, 256);
    if (tid == 0) flags[0] = grid_barrier(fa.gbar, G, fa.err, lim) ? 1 : 0;
    named_bar(1, 256);
    if (!flags[0]) {
        *abort = 1;
        __syncwarp();  // the producer still waits at barrier 4
        asm volatile("bar.arrive 4, %0;" ::"r"(32 * (PIPE_CONSUMERS + 1)) : "memory");
    } else {
        // P2: x records (async, overlapping the selection), selection, union
        for (int i = tid; i < T * rbH / 16; i += 256) cp_async16(acts + 16 * i, fa.xrec + 16 * i);
        const bool pub = blockIdx.x == 0;
        if (k == 0) {  // a dense layer: no selection; the x records, then barrier 4
            cp_async_wait_all();
            __syncwarp();
            asm volatile("bar.arrive 4, %0;" ::"r"(32 * (PIPE_CONSUMERS + 1)) : "memory");
        }
        for (int t = 0; t < T && k > 0; ++t) {
            sm.w_smem = w_s + t * k;
            // the first token's scores loaded: release the producer (barrier 4)
            cta_select_token<SyncConsumers>(fa.ws.c + (int64_t)t * E, fa.ws.s + (int64_t)t * E, E,
                                            fa.G, fa.gk, k, fa.rsf, sm, pub ? fa.ws.idx + t * k : nullptr,
                                            pub ? fa.ws.w + t * k : nullptr, idx_s + t * k, 4,
                                            t == 0 ? 32 * (PIPE_CONSUMERS + 1) : 0, fa.top_p);
        }
        if (MAXT == 1) {
            if (warp == 0) warp_union_one(lw, E, S, k, idx_s);
        } else {
            cta_union_small<SyncConsumers>(lw, T, E, S, k, cnt, idx_s, reinterpret_cast<int *>(red));
        }
        cp_async_wait_all();
        named_bar(1, 256);
        if (pub) {
            const int na = *lw.n_active, np = lw.off[na];
            for (int i = tid; i < na; i += 256) fa.ws.active[i] = lw.active[i];
            for (int i = tid; i <= na; i += 256) fa.ws.off[i] = lw.off[i];
            for (int i = tid; i < E + S; i += 256) fa.ws.act_of[i] = lw.act_of[i];
            for (int i = tid; i < np; i += 256) {
                fa.ws.pair_tok[i] = lw.pair_tok[i];
                fa.ws.pair_slot[i] = lw.pair_slot[i];
            }
            // one entry per (token, slot): more than np where slots hold -1
            for (int i = tid; i < T * (k + S); i += 256) fa.ws.tok_pair[i] = lw.tok_pair[i];
            if (tid == 0) *fa.ws.n_active = na;
        }
    }
    named_bar(2, DECODE_THREADS);        // tables ready: release producer and epilogue warp
    if (consumers_aborted(abort, flags + 1)) return;

    // down-row scales of this CTA's rows for every active expert (they need
    // no h): 4-byte async copies, landing while the gate/up items run
    const int n_active = *lw.n_active;
    {
        const int ds = fa.rows_cap + 4;
        for (int i = tid; i < n_active * nrows; i += 256) {
            const int a = i / nrows, r = i % nrows;
            const int e = lw.active[a];
            const float *dsc = fa.ptr_smem ? static_cast<const float *>(eptrs[4 * e + 3])
                                           : fa.experts[e].down.scales;
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dscale + a * ds + r)),
                         "l"(dsc + r0 + r)
                         : "memory");
        }
    }

    // P3: gate/up items; partials go to the epilogue warp through part_full /
    // part_free (two buffers)
    const FastGeo fgeo(geo, V);
    const int n_items = n_active * nchunk;
    RingPos rp;
    bool ok = true;
    int n = 0;
    // one token: the same activation for every item, loaded once
    LaneAct<BITS, 3> act1;
    if (MAXT == 1 && geo.fast) act1.load(acts, H, V, fgeo.vbase);
    for (int item = blockIdx.x; item < n_items && ok; item += G, ++n) {
        const int buf = n & 1;
        int a, e, c;
        item_expert_chunk(item, n_active, a, e, c);
        const int p0 = lw.off[a];
        const int ne = min(lw.off[a + 1] - p0, PIPE_MAX_TOK);
        const int *tok = lw.pair_tok + p0;
        const bool fast = geo.fast && (MAXT == 1 || ne == 1);
        LaneAct<BITS, 3> act;
        if (MAXT == 1) act = act1;
        else if (fast) act.load(acts + (size_t)tok[0] * rbH, H, V, fgeo.vbase);
        if (n >= 2 && !mbar_wait(&ebars->part_free[buf], (uint32_t)(((n >> 1) - 1) & 1), fa.err, lim)) {
            ok = false;
            *abort = 1;
            break;
        }
        double *pbuf = part + (size_t)buf * 2 * part_mat;
        if (fast) {
            const RingView rv{ring, bars, ns, fa.err, abort, 1, lim};
            switch (fgeo.slices) {
                case 1: ok = gateup_item_fast<BITS, 1>(rv, rp, RB, fgeo, act, pbuf, part_mat, ntok); break;
                case 2: ok = gateup_item_fast<BITS, 2>(rv, rp, RB, fgeo, act, pbuf, part_mat, ntok); break;
                default: ok = gateup_item_fast<BITS, 4>(rv, rp, RB, fgeo, act, pbuf, part_mat, ntok); break;
            }
        } else {
            for (int ms = 0; ms < steps; ++ms) {
                if (!mbar_wait(&bars->full[rp.slot], rp.phase, fa.err, lim)) {
                    ok = false;
                    *abort = 1;
                    break;
                }
                const uint8_t *stage = ring + (size_t)rp.slot * PIPE_STAGE_MAX;
                double *pm = pbuf + (ms < spm ? 0 : part_mat);
                const int row_base = (ms < spm ? ms : ms - spm) * R;
                for (int i0 = 0; i0 < ne; i0 += PIPE_PASS_TOK) {
                    const int nn = MAXT == 1 ? 1 : min(PIPE_PASS_TOK, ne - i0);
                    const int *tk = tok + i0;
                    if constexpr (MAXT == 1) {
                        gateup_stage<BITS, 1>(stage, RB, V, H, geo, row_base, acts, rbH, tk, i0, pm, ntok);
                    } else {
                        switch (nn) {
                            case 1: gateup_stage<BITS, 1>(stage, RB, V, H, geo, row_base, acts, rbH, tk, i0, pm, ntok); break;
                            case 2: gateup_stage<BITS, 2>(stage, RB, V, H, geo, row_base, acts, rbH, tk, i0, pm, ntok); break;
                            case 3: gateup_stage<BITS, 3>(stage, RB, V, H, geo, row_base, acts, rbH, tk, i0, pm, ntok); break;
                            default: gateup_stage<BITS, 4>(stage, RB, V, H, geo, row_base, acts, rbH, tk, i0, pm, ntok); break;
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->empty[rp.slot]);
                rp.next(ns);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ebars->part_full[buf]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(xfree);  // no x record is read after this
    cp_async_wait_all();
    if (consumers_aborted(abort, flags + 1)) return;
    // P4: down rows of every active expert as its h arrives, then the combine
    const int vpl = (VI % 32 == 0) ? VI / 32 : 0;
    DownLoop dl{lw.off, n_active, Sa, T, subs, ns, fa.down_rows, fa.rows_cap, r0, nrows, RBI, VI, I, rbI,
                fa.down_span, lim, ring, dscale, hslots, fa.nh, hfull, hempty, ebuf, bars, abort, fa.err};
    switch (vpl) {
        case 1: ok = down_loop<BITS, 1, MAXT>(dl, rp) && ok; break;
        case 2: ok = down_loop<BITS, 2, MAXT>(dl, rp) && ok; break;
        case 4: ok = down_loop<BITS, 4, MAXT>(dl, rp) && ok; break;
        default: ok = down_loop<BITS, 0, MAXT>(dl, rp) && ok; break;
    }
    if (consumers_aborted(abort, flags + 1)) return;
    const int slots = k + S;
    for (int q = tid; q < T * nrows; q += 256) {
        const int t = q / nrows, row = q % nrows;
        double acc = 0.0;
        for (int jj = 0; jj < slots; ++jj) {
            const int j = jj < S ? k + jj : jj - S;
            const int p = lw.tok_pair[t * slots + j];
            if (p < 0) continue;  // an expert another handle computes
            const double ev = (double)ebuf[(size_t)p * fa.rows_cap + row];
            if (j < k)
                acc = fma((double)w_s[t * k + j], ev, acc);
            else
                acc += ev;
        }
        if (fa.out_partial)
            fa.out_partial[(int64_t)t * H + r0 + row] = acc;
        else
            fa.out[(int64_t)t * H + r0 + row] = (float)acc;
    }
}

// Parity export: integer block sums of one matrix against T Q8_0 vectors.
// One warp per (token, row); lanes stride over the row's vectors.
template <int BITS>
__global__ void k_dbg_block_sums(const uint8_t *__restrict__ codes, int64_t rows, int K,
                                 const int8_t *__restrict__ xq, int T, int32_t *__restrict__ S) {
    extern __shared__ __align__(128) uint8_t smem[];
    // one token at a time staged per CTA: blockIdx.y = token
    const int t = blockIdx.y;
    uint8_t *planes = smem;
    int *xs = reinterpret_cast<int *>(smem + K);
    float *xdd = reinterpret_cast<float *>(xs + K / COLI_QBLK);
    // stage codes only (scales are not needed): reuse stage_rows with a zero scale source
    {
        constexpr int ELEMS = Fmt<BITS>::ELEMS;
        const int V = K * BITS / 128;
        for (int wd = threadIdx.x; wd < K / 4; wd += blockDim.x) {
            const int ob = wd * 4, plane = ob / (V * 16), inner = ob % (V * 16);
            const int v = inner / 16, pos = plane * 16 + (inner % 16);
            uint32_t word = 0;
#pragma unroll
            for (int b = 0; b < 4; ++b)
                word |= (uint32_t)(uint8_t)xq[(int64_t)t * K + v * ELEMS + stage_src<BITS>(pos + b)]
                        << (8 * b);
            reinterpret_cast<uint32_t *>(planes)[wd] = word;
        }
        for (int b = threadIdx.x; b < K / COLI_QBLK; b += blockDim.x) {
            int sum = 0;
            for (int j = 0; j < COLI_QBLK; ++j) sum += xq[(int64_t)t * K + b * COLI_QBLK + j];
            xs[b] = sum;
            xdd[b] = 0.0f;
        }
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    const int V = K * BITS / 128;
    const int nb = K / COLI_QBLK;
    const int64_t rowbytes = (int64_t)K * BITS / 8;
    for (int64_t r = (int64_t)blockIdx.x * nwarps + warp; r < rows; r += (int64_t)gridDim.x * nwarps) {
        const uint4 *row = reinterpret_cast<const uint4 *>(codes + r * rowbytes);
        int32_t *Sr = S + ((int64_t)t * rows + r) * nb;
        for (int b = lane; b < nb; b += 32) Sr[b] = 0;
        __syncwarp();
        for (int v = lane; v < V; v += 32) {
            int s0, s1, b0, S0, b1, S1;
            vec_dot<BITS>(ldg_stream(row + v), reinterpret_cast<const uint4 *>(planes) + v, V, s0, s1);
            vec_block_sums<BITS>(v, s0, s1, xs, b0, S0, b1, S1);
            atomicAdd(Sr + b0, S0);
            if (b1 >= 0) atomicAdd(Sr + b1, S1);
        }
        __syncwarp();
    }
}

}  // namespace coli
