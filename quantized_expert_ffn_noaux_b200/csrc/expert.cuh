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
                          int S, float *__restrict__ out) {
    const int64_t n = (int64_t)T * H;
    const int slots = k + S;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int t = (int)(i / H), r = (int)(i % H);
        double acc = 0.0;
        for (int jj = 0; jj < slots; ++jj) {
            const int j = jj < S ? k + jj : jj - S;
            const int p = ws.tok_pair[(int64_t)t * slots + j];
            const double ev = (double)e_pairs[(int64_t)p * H + r];
            if (j < k)
                acc = fma((double)ws.w[(int64_t)t * k + j], ev, acc);
            else
                acc += ev;
        }
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
                                                      float *__restrict__ out) {
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
                const double ev = ep[(size_t)p * DOWN_ROWS + rr];
                if (j < k)
                    acc = fma((double)ws.w[(int64_t)t * k + j], ev, acc);
                else
                    acc += ev;
            }
            out[(int64_t)t * H + r0 + rr] = (float)acc;
        }
        __syncwarp();
    }
}

// ===========================================================================
// Few-token (decode / verification) kernels: weight rows stream through a
// shared-memory ring with cp.async.bulk copies issued by one producer thread
// and completed on mbarriers; sixteen consumer warps run the integer dots out
// of shared memory.  One CTA per SM, persistent.  Every wait is bounded: on a
// timeout the kernel records COLI_ETIMEOUT in *err, drains its own copies and
// returns.
constexpr int PIPE_CONSUMERS = 16;
constexpr int PIPE_THREADS = 32 * (PIPE_CONSUMERS + 1);
constexpr int PIPE_STAGE_MAX = 48 * 1024;  // bytes of weights per ring stage (at most)
constexpr int PIPE_MAX_STAGES = 8;
constexpr int PIPE_MAX_TOK = 8;            // tokens per expert on the few-token path
constexpr int PIPE_PASS_TOK = 4;           // tokens per pass over a staged weight row

struct PipeBars {
    uint64_t full[PIPE_MAX_STAGES];
    uint64_t empty[PIPE_MAX_STAGES];
    uint64_t act;
    int abort;
};

__host__ __device__ inline size_t pipe_hdr_bytes() { return (sizeof(PipeBars) + 127) & ~(size_t)127; }
__host__ __device__ inline size_t align128(size_t x) { return (x + 127) & ~(size_t)127; }

// Gate/up rows per stage: a power of two dividing 32 with R * rowbytes <= 48 KB.
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

// Gate/up consumer work for one stage: row slices assigned to this warp,
// NT tokens; writes the reduced sums to part[row][slice][token].
template <int BITS, int NT>
__device__ __forceinline__ void gateup_stage(const uint8_t *stage, int RB, int V, int H, int R,
                                             int slices, int rows_per_warp, int row_base,
                                             const uint8_t *acts, int rbH, const int *tok,
                                             int i0, double *part_mat) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint8_t *rec[NT];
#pragma unroll
    for (int i = 0; i < NT; ++i) rec[i] = acts + (size_t)tok[i] * rbH;
    for (int rr = 0; rr < rows_per_warp; ++rr) {
        const int row = (slices == 1) ? warp * rows_per_warp + rr : warp / slices;
        const int sl = (slices == 1) ? 0 : warp % slices;
        const int v_lo = (int)((long long)sl * V / slices);
        const int v_hi = (int)((long long)(sl + 1) * V / slices);
        double acc[NT];
        slice_dot<BITS, NT>(reinterpret_cast<const uint4 *>(stage + (size_t)row * RB), v_lo, v_hi, V,
                            H, rec, acc);
#pragma unroll
        for (int i = 0; i < NT; ++i) {
            const double tot = warp_sum(acc[i]);
            if (lane == 0) part_mat[((row_base + row) * slices + sl) * PIPE_MAX_TOK + i0 + i] = tot;
        }
    }
}

// Gate/up of the few-token path, fused with SwiGLU and Q8_0(h).
// Items: (active expert, 32-row chunk of the intermediate); each item streams
// the chunk's gate rows, then its up rows, R rows per stage.  The partial sums
// of an item are double-buffered so the SwiGLU/Q8_0 epilogue of item n runs
// while the next item's stages are consumed; one named barrier per item.
// Dynamic smem: PipeBars | tables | T activation records | ring | partials.
template <int BITS>
__global__ void __launch_bounds__(PIPE_THREADS, 1)
    k_gateup_pipe(RouteWs ws, const ExpertDev *__restrict__ experts,
                  const uint8_t *__restrict__ xrec, int T, int H, int I, int ns, int amax,
                  int npairs_max, uint8_t *__restrict__ hrec, int8_t *__restrict__ hq, float *__restrict__ hd,
                  int *__restrict__ err) {
    extern __shared__ __align__(128) uint8_t smem[];
    PipeBars *bars = reinterpret_cast<PipeBars *>(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int RB = H * BITS / 8;                 // bytes per weight row
    const int V = H * BITS / 128;                // uint4 vectors per row
    const int R = pipe_rows_per_stage(RB);       // rows per stage
    const int spm = 32 / R;                      // stages per matrix per item
    const int nchunk = I / 32;
    const int rbH = rec_bytes(H);
    const int slices = R >= PIPE_CONSUMERS ? 1 : PIPE_CONSUMERS / R;
    const int rows_per_warp = R >= PIPE_CONSUMERS ? R / PIPE_CONSUMERS : 1;
    int *t_active = reinterpret_cast<int *>(smem + pipe_hdr_bytes());
    int *t_off = t_active + amax;
    int *t_tok = t_off + amax + 1;
    uint8_t *acts = smem + pipe_hdr_bytes() + align128((size_t)(2 * amax + 1 + npairs_max) * 4);
    uint8_t *ring = acts + align128((size_t)T * rbH);
    const size_t stage_bytes = (size_t)R * RB;
    double *part = reinterpret_cast<double *>(ring + (size_t)ns * stage_bytes);
    const size_t part_mat = (size_t)32 * slices * PIPE_MAX_TOK;  // doubles per (buffer, matrix)
    pipe_init(bars, ns);
    pdl_wait();
    const int n_active = *ws.n_active;
    const int n_pairs = ws.off[n_active];
    for (int i = tid; i < n_active; i += blockDim.x) t_active[i] = ws.active[i];
    for (int i = tid; i <= n_active; i += blockDim.x) t_off[i] = ws.off[i];
    for (int i = tid; i < n_pairs; i += blockDim.x) t_tok[i] = ws.pair_tok[i];
    __syncthreads();
    pdl_launch_dependents();
    const int n_items = n_active * nchunk;
    const int steps = 2 * spm;
    if (warp == PIPE_CONSUMERS) {
        if (lane != 0) return;
        // ------------------------------ producer
        mbar_expect_tx(&bars->act, (uint32_t)(T * rbH));
        bulk_g2s(acts, xrec, (uint32_t)(T * rbH), &bars->act);
        long long s = 0;
        for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
            const int a = item / nchunk, c = item % nchunk;
            const ExpertDev ex = experts[t_active[a]];
            for (int ms = 0; ms < steps; ++ms, ++s) {
                const int slot = (int)(s % ns);
                if (s >= ns && !mbar_wait(&bars->empty[slot], (uint32_t)(((s / ns) - 1) & 1), err)) {
                    pipe_drain(bars, ns, s, s - ns, err);
                    mbar_wait(&bars->act, 0, err);
                    return;
                }
                const QMatDev M = (ms < spm) ? ex.gate : ex.up;
                const int row0 = c * 32 + (ms % spm) * R;
                mbar_expect_tx(&bars->full[slot], (uint32_t)stage_bytes);
                bulk_g2s(ring + (size_t)slot * stage_bytes, M.codes + (size_t)row0 * RB,
                         (uint32_t)stage_bytes, &bars->full[slot]);
            }
        }
        return;  // the consumers wait for every copy
    }
    // ---------------------------------- consumers
    // A timed-out wait sets bars->abort; every consumer warp still passes each
    // named barrier, and all of them leave together right after one.
    volatile int *abort = &bars->abort;
    bool ok = mbar_wait(&bars->act, 0, err);
    if (!ok) *abort = 1;
    long long s = 0;
    int buf = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x, buf ^= 1) {
        const int a = item / nchunk, c = item % nchunk;
        const int p0 = t_off[a];
        const int ne = min(t_off[a + 1] - p0, PIPE_MAX_TOK);
        const int *tok = t_tok + p0;
        // the epilogue warps fetch their row scales early
        float sg = 0.0f, su = 0.0f;
        const ExpertDev ex = experts[t_active[a]];
        if (warp < ne) {
            sg = __ldg(ex.gate.scales + c * 32 + lane);
            su = __ldg(ex.up.scales + c * 32 + lane);
        }
        double *pbuf = part + (size_t)buf * 2 * part_mat;
        for (int ms = 0; ms < steps && ok; ++ms, ++s) {
            const int slot = (int)(s % ns);
            if (!mbar_wait(&bars->full[slot], (uint32_t)((s / ns) & 1), err)) {
                ok = false;
                *abort = 1;
                break;
            }
            const uint8_t *stage = ring + (size_t)slot * stage_bytes;
            double *pm = pbuf + (ms < spm ? 0 : part_mat);
            const int row_base = (ms % spm) * R;
            // tokens in passes of at most PIPE_PASS_TOK over the staged rows
            for (int i0 = 0; i0 < ne; i0 += PIPE_PASS_TOK) {
                const int n = min(PIPE_PASS_TOK, ne - i0);
                const int *tk = tok + i0;
                switch (n) {
                    case 1: gateup_stage<BITS, 1>(stage, RB, V, H, R, slices, rows_per_warp, row_base, acts, rbH, tk, i0, pm); break;
                    case 2: gateup_stage<BITS, 2>(stage, RB, V, H, R, slices, rows_per_warp, row_base, acts, rbH, tk, i0, pm); break;
                    case 3: gateup_stage<BITS, 3>(stage, RB, V, H, R, slices, rows_per_warp, row_base, acts, rbH, tk, i0, pm); break;
                    default: gateup_stage<BITS, 4>(stage, RB, V, H, R, slices, rows_per_warp, row_base, acts, rbH, tk, i0, pm); break;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->empty[slot]);
        }
        named_bar(1, 32 * PIPE_CONSUMERS);
        if (*abort) break;
        // SwiGLU + Q8_0(h) of this item: warp i handles token i, lane = row in chunk
        if (warp < ne) {
            const int i = warp;
            double ag = 0.0, au = 0.0;
            for (int sl = 0; sl < slices; ++sl) {
                ag += pbuf[((size_t)lane * slices + sl) * PIPE_MAX_TOK + i];
                au += pbuf[part_mat + ((size_t)lane * slices + sl) * PIPE_MAX_TOK + i];
            }
            const float g = (float)(ag * (double)sg);
            const float u = (float)(au * (double)su);
            const double gd = (double)g;
            const float h = (float)((gd / (1.0 + exp(-gd))) * (double)u);
            const int p = p0 + i;
            q8_block_to_record<BITS>(h, c, I, hrec + (size_t)p * rec_bytes(I), hq + (int64_t)p * I,
                                     hd + (int64_t)p * (I / COLI_QBLK));
        }
    }
}

// Down consumer work for one stage: rows w, w+16, ... of the stage, NT tokens
// starting at pair p; writes e = (float)(sum * row scale) to ebuf.
template <int BITS, int NT>
__device__ __forceinline__ void down_stage(const uint8_t *stage, int RB, int V, int I, int nr,
                                           const float *scales, const uint8_t *hacts, int rbI,
                                           int p, float *ebuf, int rows_cap, int row_off) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint8_t *rec[NT];
#pragma unroll
    for (int i = 0; i < NT; ++i) rec[i] = hacts + (size_t)(p + i) * rbI;
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

// Down projection + combine of the few-token path.  CTA b owns a contiguous
// range of output rows (balanced over the grid) and streams, for every active
// expert in order, those rows of its down matrix; e values land in shared
// memory and the CTA combines each token's slots in the fixed order (shared
// experts first, then routed slots) in fp64.
// Dynamic smem: PipeBars | all pairs' h records | ring | e values | row scales.
template <int BITS>
__global__ void __launch_bounds__(PIPE_THREADS, 1)
    k_down_pipe(RouteWs ws, const ExpertDev *__restrict__ experts,
                const uint8_t *__restrict__ hrec, int T, int H, int I, int k, int S, int ns,
                int stage_rows, int rows_cap, float *__restrict__ out, int *__restrict__ err) {
    extern __shared__ __align__(128) uint8_t smem[];
    PipeBars *bars = reinterpret_cast<PipeBars *>(smem);
    const int rbI = rec_bytes(I);
    const int n_pairs_max = T * (k + S);
    const int RB = I * BITS / 8;
    const int V = I * BITS / 128;
    const size_t stage_bytes = (size_t)stage_rows * RB;
    uint8_t *hacts = smem + pipe_hdr_bytes();
    uint8_t *ring = hacts + align128((size_t)n_pairs_max * rbI);
    float *ebuf = reinterpret_cast<float *>(ring + (size_t)ns * stage_bytes);  // [pairs][rows_cap]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int base = H / gridDim.x, rem = H % gridDim.x;
    const int r0 = blockIdx.x * base + min((int)blockIdx.x, rem);
    const int nrows = base + ((int)blockIdx.x < rem ? 1 : 0);
    pipe_init(bars, ns);
    __syncthreads();
    // The routing tables were complete before the gate/up kernel started, so
    // the producer may stream down weights before the gate/up grid finishes;
    // the h records are read only after pdl_wait.
    const int n_active = *ws.n_active;
    const int subs = (nrows + stage_rows - 1) / stage_rows;
    if (warp == PIPE_CONSUMERS) {
        if (lane != 0) return;
        long long s = 0;
        bool act_issued = false;
        auto issue_act = [&]() {
            pdl_wait();
            const int n_pairs = ws.off[n_active];
            mbar_expect_tx(&bars->act, (uint32_t)(n_pairs * rbI));
            bulk_g2s(hacts, hrec, (uint32_t)(n_pairs * rbI), &bars->act);
            act_issued = true;
        };
        for (int a = 0; a < n_active; ++a) {
            const QMatDev M = experts[ws.active[a]].down;
            for (int sb = 0; sb < subs; ++sb, ++s) {
                const int slot = (int)(s % ns);
                if (s >= ns) {
                    // the ring is full: the consumers need the h records to free it
                    if (!act_issued) issue_act();
                    if (!mbar_wait(&bars->empty[slot], (uint32_t)(((s / ns) - 1) & 1), err)) {
                        pipe_drain(bars, ns, s, s - ns, err);
                        mbar_wait(&bars->act, 0, err);
                        return;
                    }
                }
                const int rs = r0 + sb * stage_rows;
                const int nr = min(stage_rows, r0 + nrows - rs);
                mbar_expect_tx(&bars->full[slot], (uint32_t)(nr * RB));
                bulk_g2s(ring + (size_t)slot * stage_bytes, M.codes + (size_t)rs * RB,
                         (uint32_t)(nr * RB), &bars->full[slot]);
            }
        }
        if (!act_issued) issue_act();
        return;
    }
    pdl_wait();
    pdl_launch_dependents();
    volatile int *abort = &bars->abort;
    bool ok = mbar_wait(&bars->act, 0, err);
    if (!ok) *abort = 1;
    long long s = 0;
    for (int a = 0; a < n_active && ok; ++a) {
        const QMatDev M = experts[ws.active[a]].down;
        const int p0 = ws.off[a], ne = ws.off[a + 1] - p0;
        for (int sb = 0; sb < subs; ++sb, ++s) {
            const int slot = (int)(s % ns);
            if (!mbar_wait(&bars->full[slot], (uint32_t)((s / ns) & 1), err)) {
                ok = false;
                *abort = 1;
                break;
            }
            const int rs = r0 + sb * stage_rows;
            const int nr = min(stage_rows, r0 + nrows - rs);
            const uint8_t *stage = ring + (size_t)slot * stage_bytes;
            for (int i0 = 0; i0 < ne; i0 += PIPE_PASS_TOK) {
                const int n = min(PIPE_PASS_TOK, ne - i0);
                const float *sc = M.scales + rs;
                const int ro = rs - r0;
                switch (n) {
                    case 1: down_stage<BITS, 1>(stage, RB, V, I, nr, sc, hacts, rbI, p0 + i0, ebuf, rows_cap, ro); break;
                    case 2: down_stage<BITS, 2>(stage, RB, V, I, nr, sc, hacts, rbI, p0 + i0, ebuf, rows_cap, ro); break;
                    case 3: down_stage<BITS, 3>(stage, RB, V, I, nr, sc, hacts, rbI, p0 + i0, ebuf, rows_cap, ro); break;
                    default: down_stage<BITS, 4>(stage, RB, V, I, nr, sc, hacts, rbI, p0 + i0, ebuf, rows_cap, ro); break;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->empty[slot]);
        }
    }
    named_bar(1, 32 * PIPE_CONSUMERS);
    if (*abort) return;
    const int slots = k + S;
    for (int q = tid; q < T * nrows; q += 32 * PIPE_CONSUMERS) {
        const int t = q / nrows, row = q % nrows;
        double acc = 0.0;
        for (int jj = 0; jj < slots; ++jj) {
            const int j = jj < S ? k + jj : jj - S;
            const int p = ws.tok_pair[t * slots + j];
            const double ev = (double)ebuf[(size_t)p * rows_cap + row];
            if (j < k)
                acc = fma((double)ws.w[t * k + j], ev, acc);
            else
                acc += ev;
        }
        out[(int64_t)t * H + r0 + row] = (float)acc;
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
