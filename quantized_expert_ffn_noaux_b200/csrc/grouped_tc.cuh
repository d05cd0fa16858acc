// Many-token expert GEMMs on the 5th-generation tensor cores.
//
// Batch-union prefill ("Sparse MoE: batch-union routing" and "Int8/int4
// quantised matmul with Q8_0 activations" in the engine write-up): the tokens
// routed to an expert are gathered into one grouped GEMM per expert.  The
// Q8_0 dot has one activation scale per 32-wide block of K, so a tile's
// integer products are needed block by block: each block is one
// tcgen05.mma kind::i8 (M = 128 weight rows, N = 32 tokens, K = 32) into its
// own TMEM accumulator, and epilogue warps promote it exactly as the scalar
// definition does -- acc += (double)S_b * (double)d_b in fp64, then
// value = (float)(acc * row_scale).
//
// One CTA per SM, persistent over items (active expert, row tile, 32-token
// tile), 24 warps:
//   warp 0      producer: four 2-D TMA copies a stage of 8 blocks -- the two
//               128-row tiles of raw weight codes (int8/int4/int2), and the 32
//               pair rows of activation codes and of block scales (pair order:
//               x is gathered by pair first, h is written that way)
//   warp 1      TMEM owner; one thread issues the two MMAs of a block
//   warps 2, 3, 20-23   expand one block at a time into the K-major
//               canonical layout, scales to fp64
//   warps 4-19  epilogue: warp 4 + q + 4 m + 8 h reads TMEM lane quarter q
//               of A tile m, token columns 16 h .. 16 h + 15; exact fp64
//               promotion (the fp64 pipe bounds the kernel); the item's end
// Gate/up items pair the gate and up rows of a 128-row tile and end in
// SwiGLU + Q8_0(h); down items pair two 128-row tiles of the down matrix and
// end in the per-pair outputs e[p][row].  Every wait is bounded.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "route.cuh"
#include "expert.cuh"

namespace coli {

constexpr int TC_M = 128;        // weight rows per A tile
constexpr int TC_N = 32;         // tokens per item
constexpr int TC_BPS = 8;        // 32-blocks per stage
constexpr int TC_STAGES = 2;     // raw stages
constexpr int TC_SLOTS = 4;      // canonical operand slots (one block each)
constexpr int TC_BUFS = 4;       // TMEM accumulator buffers (64 columns each) and scale slots
constexpr int TC_THREADS = 768;
constexpr int TC_EXPAND_WARPS = 6;  // warps 2, 3 and 20-23
constexpr int TC_EPI_WARPS = 16;    // warps 4-19
constexpr int TC_EXPAND_THREADS = 32 * TC_EXPAND_WARPS;
constexpr int TC_EXPAND_GROUP = TC_EXPAND_THREADS / 2;  // two groups take alternate blocks
constexpr int TC_TMEM_COLS = 256;
constexpr int TC_OP_BYTES = 2 * TC_M * 32 + TC_N * 32;  // A0, A1, B of one block
// Raw weight codes land block-major: column groups of tc_group_bytes(BITS)
// bytes (one 32-block, two for int2) of all 128 rows, so that the expanding
// lanes read consecutive rows (no bank conflicts).
__host__ __device__ constexpr int tc_group_bytes(int bits) { return 4 * bits < 16 ? 16 : 4 * bits; }

struct TcBars {
    uint64_t raw_full[TC_STAGES], raw_empty[TC_STAGES];
    uint64_t op_full[TC_SLOTS], op_empty[TC_SLOTS];
    uint64_t tm_full[TC_BUFS], tm_empty[TC_BUFS];
    uint64_t dd_full[TC_BUFS], dd_empty[TC_BUFS];
    uint32_t taddr;
    int abort;
    int n_items;
    int pad;
    int pair_ok[16];   // gate/up epilogue pairs: each warp's ok, exchanged at the item's end
};

struct TcLayout {
    size_t bars, starts, raw, op, dd, xch, total;
    int rawA, rawB, rawD, raw_stage;
};

// Shared-memory layout for a weight format (raw A rows of 8 blocks).
__host__ __device__ inline TcLayout tc_layout(int bits, int max_active) {
    TcLayout L;
    size_t o = 0;
    L.bars = o;
    o += (sizeof(TcBars) + 127) & ~(size_t)127;
    L.starts = o;                                      // item prefix per active expert
    o += (((size_t)max_active + 1) * 4 + 127) & ~(size_t)127;
    L.rawA = 2 * TC_M * TC_BPS * 32 * bits / 8;
    L.rawB = TC_N * TC_BPS * 32;
    L.rawD = TC_N * TC_BPS * 4;
    L.raw_stage = L.rawA + L.rawB + L.rawD;
    L.raw = o;
    o += (size_t)TC_STAGES * L.raw_stage;
    o = (o + 127) & ~(size_t)127;
    L.op = o;
    o += (size_t)TC_SLOTS * TC_OP_BYTES;
    L.dd = o;
    o += (size_t)TC_BUFS * TC_N * 8;
    L.xch = o;                                         // u, then g, of the 4 lane quarters
    o += (size_t)2 * 4 * TC_N * 32 * 4;
    L.total = o;
    return L;
}

// Tensor maps, in one device array: activations first, then gate, up and down
// of every expert (expert e, matrix m at TC_MAP_W + 3 e + m).
constexpr int TC_MAP_XG = 0, TC_MAP_XD = 1, TC_MAP_HQ = 2, TC_MAP_HD = 3, TC_MAP_W = 4;

struct TcArgs {
    RouteWs ws;
    const ExpertDev *experts;
    const CUtensorMap *maps;
    int down;               // 0: gate/up items, 1: down items
    int K;                  // reduction length (H for gate/up, I for down)
    int I;                  // intermediate size (h layout)
    int H;                  // hidden size (e_pairs layout)
    int map_b, map_d;       // maps of the activation codes and scales [pairs][K], [pairs][K/32]
    const double *corr;     // per pair: the weight offset's share (int4 / int2), see k_pair_offsets
    int8_t *hq;             // gate/up outputs
    float *hd;
    float *e_pairs;         // down output [pairs][H]
    int *err;
    const long long *wait_limit;  // SM cycles a wait on progress may last (drains keep the default)
};

// --- tcgen05 wrappers -------------------------------------------------------
__device__ __forceinline__ uint64_t tc_desc(uint32_t saddr) {
    // K-major, no swizzle: core matrices of 8 rows x 16 bytes, the two 16-byte
    // halves of a 32-byte K block 128 bytes apart (leading byte offset), row
    // groups of 8 rows 256 bytes apart (stride byte offset); version 1.
    return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)(128 >> 4) << 16) |
           ((uint64_t)(256 >> 4) << 32) | (1ull << 46);
}
// kind::i8, s32 accumulator, K-major A and B, M = 128, N = TC_N; B (the
// activation codes) signed, A signed for int8 weights and unsigned for int4 /
// int2 (codes stored as code + 8 / code + 2, see tc_expand)
template <int BITS>
__host__ __device__ constexpr uint32_t tc_idesc() {
    return (2u << 4) | ((BITS == 8 ? 1u : 0u) << 7) | (1u << 10) | ((uint32_t)(TC_N >> 3) << 17) |
           ((uint32_t)(TC_M >> 4) << 24);
}

template <int BITS>
__device__ __forceinline__ void tc_mma(uint32_t dtmem, uint64_t da, uint64_t db) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}\n" ::"r"(dtmem),
        "l"(da), "l"(db), "r"(tc_idesc<BITS>()), "r"(0u));
}
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

__device__ __forceinline__ void tma2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"((uint64_t)map), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Activation codes and block scales of every (token, expert) pair in pair
// order, so that a tile of 32 pairs is one 2-D box.
__global__ void k_gather_pairs(RouteWs ws, const int8_t *__restrict__ xq, const float *__restrict__ xd,
                               int H, int8_t *__restrict__ xg, float *__restrict__ xdg) {
    const int np = ws.off[*ws.n_active];
    const int nb = H / COLI_QBLK;
    for (int p = blockIdx.x; p < np; p += gridDim.x) {
        const int t = ws.pair_tok[p];
        const uint4 *src = reinterpret_cast<const uint4 *>(xq + (size_t)t * H);
        uint4 *dst = reinterpret_cast<uint4 *>(xg + (size_t)p * H);
        for (int i = threadIdx.x; i < H / 16; i += blockDim.x) dst[i] = src[i];
        for (int i = threadIdx.x; i < nb; i += blockDim.x) xdg[(size_t)p * nb + i] = xd[(size_t)t * nb + i];
    }
}

// Per pair, the unsigned-weight offset's share of every row's sum:
// off * sum_b (sum of the pair's codes in block b) * d_b, in fp64, blocks in
// order (deterministic).  One CTA per pair; codes [pairs][K] in pair order.
__global__ void __launch_bounds__(256) k_pair_offsets(RouteWs ws, const int8_t *__restrict__ q,
                                                      const float *__restrict__ d, int K, double off,
                                                      double *__restrict__ out) {
    // one warp per pair: lanes stride over the blocks, one fp64 warp sum
    const int np = ws.off[*ws.n_active];
    const int nb = K / COLI_QBLK;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int p = (int)blockIdx.x * 8 + warp; p < np; p += (int)gridDim.x * 8) {
        double acc = 0.0;
        for (int b = lane; b < nb; b += 32) {
            const int4 *c = reinterpret_cast<const int4 *>(q + (size_t)p * K + (size_t)b * COLI_QBLK);
            const int4 c0 = c[0], c1 = c[1];
            int sx = 0;
            sx = __dp4a(c0.x, 0x01010101, sx);
            sx = __dp4a(c0.y, 0x01010101, sx);
            sx = __dp4a(c0.z, 0x01010101, sx);
            sx = __dp4a(c0.w, 0x01010101, sx);
            sx = __dp4a(c1.x, 0x01010101, sx);
            sx = __dp4a(c1.y, 0x01010101, sx);
            sx = __dp4a(c1.z, 0x01010101, sx);
            sx = __dp4a(c1.w, 0x01010101, sx);
            acc = fma((double)sx, (double)d[(size_t)p * nb + b], acc);
        }
        acc = warp_sum(acc);
        if (lane == 0) out[p] = off * acc;
    }
}

// Bounded wait that also gives up once another role has aborted.
__device__ __forceinline__ bool tc_wait(uint64_t *bar, uint32_t parity, TcBars *tb, int *err,
                                        long long lim) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*(volatile int *)&tb->abort) return false;
        if (clock64() - t0 > lim) {
            atomicExch(err, ERR_TIMEOUT);
            *(volatile int *)&tb->abort = 1;
            return false;
        }
    }
}

// One weight row's 32-wide block, raw codes -> 32 MMA operand bytes (two
// 16-byte halves of the canonical layout).  Element k of a row: int8 byte k
// (signed, as is); int4 nibble k (low nibble first) as the unsigned code + 8;
// int2 crumb k (low bits first) as the unsigned code + 2.  The offset's
// contribution, off * sum_k x_k per block, is removed per pair at the end
// (tc_pair_offsets).
template <int BITS>
__device__ __forceinline__ void tc_expand(const uint8_t *raw, uint4 &c0, uint4 &c1) {
    if constexpr (BITS == 8) {
        c0 = *reinterpret_cast<const uint4 *>(raw);
        c1 = *reinterpret_cast<const uint4 *>(raw + 16);
    } else if constexpr (BITS == 4) {
        const uint4 w = *reinterpret_cast<const uint4 *>(raw);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
        uint32_t o[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            // nibble v (two's complement) -> v ^ 8 = code + 8
            const uint32_t lo = (ws[i] & 0x0F0F0F0Fu) ^ 0x08080808u;
            const uint32_t hi = ((ws[i] >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
            o[2 * i] = prmt(lo, hi, 0x5140);      // elements 8i+0..3
            o[2 * i + 1] = prmt(lo, hi, 0x7362);  // elements 8i+4..7
        }
        c0 = make_uint4(o[0], o[1], o[2], o[3]);
        c1 = make_uint4(o[4], o[5], o[6], o[7]);
    } else {
        const uint2 w = *reinterpret_cast<const uint2 *>(raw);
        const uint32_t ws[2] = {w.x, w.y};
        uint32_t o[8];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            uint32_t c[4];
#pragma unroll
            for (int s = 0; s < 4; ++s)
                c[s] = ((ws[i] >> (2 * s)) & 0x03030303u) ^ 0x02020202u;  // code + 2
            const uint32_t t01l = prmt(c[0], c[1], 0x5140), t23l = prmt(c[2], c[3], 0x5140);
            const uint32_t t01h = prmt(c[0], c[1], 0x7362), t23h = prmt(c[2], c[3], 0x7362);
            o[4 * i + 0] = prmt(t01l, t23l, 0x5410);
            o[4 * i + 1] = prmt(t01l, t23l, 0x7632);
            o[4 * i + 2] = prmt(t01h, t23h, 0x5410);
            o[4 * i + 3] = prmt(t01h, t23h, 0x7632);
        }
        c0 = make_uint4(o[0], o[1], o[2], o[3]);
        c1 = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

__device__ __forceinline__ uint32_t tc_canon(int r, int half) {
    return (uint32_t)((r >> 3) * 256 + half * 128 + (r & 7) * 16);
}

template <int BITS>
__global__ void __launch_bounds__(TC_THREADS, 1) k_grouped_tc(const __grid_constant__ TcArgs a) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_active = *a.ws.n_active;
    const long long lim = *a.wait_limit;
    const TcLayout L = tc_layout(BITS, n_active);
    TcBars *tb = reinterpret_cast<TcBars *>(smem + L.bars);
    int *starts = reinterpret_cast<int *>(smem + L.starts);
    const int rows_total = a.down ? a.H : a.I;            // rows of the weight matrices
    const int RT = a.down ? rows_total / (2 * TC_M) : rows_total / TC_M;
    const int nblk = a.K / 32;                            // blocks per item
    const int nstage = nblk / TC_BPS;
    const int rawrow = TC_BPS * 32 * BITS / 8;            // raw bytes of a row per stage

    if (tid == 0) {
        for (int i = 0; i < TC_STAGES; ++i) {
            mbar_init(&tb->raw_full[i], 1);
            mbar_init(&tb->raw_empty[i], TC_EXPAND_WARPS);
        }
        for (int i = 0; i < TC_SLOTS; ++i) {
            mbar_init(&tb->op_full[i], TC_EXPAND_WARPS / 2);
            mbar_init(&tb->op_empty[i], 1);
        }
        for (int i = 0; i < TC_BUFS; ++i) {
            mbar_init(&tb->tm_full[i], 1);
            mbar_init(&tb->tm_empty[i], TC_EPI_WARPS);
            mbar_init(&tb->dd_full[i], TC_EXPAND_WARPS / 2);
            mbar_init(&tb->dd_empty[i], TC_EPI_WARPS);
        }
        tb->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // item prefix over the active experts (warp 0): items of expert a =
    // RT * ceil(ne_a / TC_N), in order (row tile, token tile fastest)
    if (warp == 0) {
        int run = 0;
        for (int b = 0; b < n_active; b += 32) {
            const int e = b + lane;
            const int ne = e < n_active ? a.ws.off[e + 1] - a.ws.off[e] : 0;
            int v = RT * ((ne + TC_N - 1) / TC_N);
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += n;
            }
            if (e < n_active) starts[e + 1] = run + v;
            run += __shfl_sync(0xffffffffu, v, 31);
        }
        if (lane == 0) {
            starts[0] = 0;
            tb->n_items = run;
        }
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&tb->taddr)),
                     "r"(TC_TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tb->taddr;
    const int n_items = tb->n_items;

    // item -> (active expert, row tile, token tile)
    auto decode_item = [&](int item, int &ae, int &rt, int &tt) {
        int lo = 0, hi = n_active - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (starts[mid] <= item) lo = mid;
            else hi = mid - 1;
        }
        ae = lo;
        const int ne = a.ws.off[ae + 1] - a.ws.off[ae];
        const int ntt = (ne + TC_N - 1) / TC_N;
        const int local = item - starts[ae];
        rt = local / ntt;
        tt = local - rt * ntt;
    };
    // A tile m of an item: its row scales, first row and tensor map
    auto a_rows = [&](int ae, int rt, int m, const float *&scales, int &row0, int &map) {
        const int e = a.ws.active[ae];
        const ExpertDev ex = a.experts[e];
        if (a.down) {
            scales = ex.down.scales;
            row0 = rt * 2 * TC_M + m * TC_M;
            map = TC_MAP_W + 3 * e + 2;
        } else {
            scales = m ? ex.up.scales : ex.gate.scales;
            row0 = rt * TC_M;
            map = TC_MAP_W + 3 * e + m;
        }
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        int sc = 0;
        if (lane == 0) {
            bool ok = true;
            for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
                int ae, rt, tt;
                decode_item(item, ae, rt, tt);
                const int p0 = a.ws.off[ae] + tt * TC_N;
                int r0[2], mp[2];
                for (int m = 0; m < 2; ++m) {
                    const float *s_unused;
                    a_rows(ae, rt, m, s_unused, r0[m], mp[m]);
                }
                for (int s = 0; s < nstage; ++s, ++sc) {
                    const int slot = sc % TC_STAGES;
                    const uint32_t ph = (uint32_t)(sc / TC_STAGES) & 1u;
                    if (!tc_wait(&tb->raw_empty[slot], ph ^ 1u, tb, a.err, lim)) {
                        ok = false;
                        break;
                    }
                    uint8_t *raw = smem + L.raw + (size_t)slot * L.raw_stage;
                    uint64_t *bar = &tb->raw_full[slot];
                    mbar_expect_tx(bar, (uint32_t)(L.rawA + L.rawB + L.rawD));
                    const int k0 = s * TC_BPS * 32;  // first element of the stage
                    constexpr int GB = tc_group_bytes(BITS);
#pragma unroll
                    for (int m = 0; m < 2; ++m)
                        for (int g = 0; g < rawrow / GB; ++g)
                            tma2d(raw + (size_t)m * TC_M * rawrow + (size_t)g * TC_M * GB, a.maps + mp[m],
                                  k0 * BITS / 8 + g * GB, r0[m], bar);
                    for (int j = 0; j < TC_BPS; ++j)
                        tma2d(raw + L.rawA + j * (TC_N * 32), a.maps + a.map_b, k0 + 32 * j, p0, bar);
                    tma2d(raw + L.rawA + L.rawB, a.maps + a.map_d, k0 / COLI_QBLK, p0, bar);
                }
            }
            // drain: every issued stage must land before the CTA leaves
            for (int d = max(0, sc - TC_STAGES); d < sc; ++d) {
                const int slot = d % TC_STAGES;
                const uint32_t ph = (uint32_t)(d / TC_STAGES) & 1u;
                if (!mbar_wait(&tb->raw_full[slot], ph, a.err)) break;
            }
        }
        __syncwarp();
    } else if (warp == 2 || warp == 3 || warp >= 4 + TC_EPI_WARPS) {
        // ------------------------------------------------------------ expand
        const int et = warp < 4 ? tid - 64 : tid - 32 * (4 + TC_EPI_WARPS) + 64;  // 0..191
        const int grp = et / TC_EXPAND_GROUP, gt = et % TC_EXPAND_GROUP;        // whole warps per group
        int sc = 0, blk = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
            for (int s = 0; s < nstage && ok; ++s, ++sc) {
                const int slot = sc % TC_STAGES;
                if (!tc_wait(&tb->raw_full[slot], (uint32_t)(sc / TC_STAGES) & 1u, tb, a.err, lim)) {
                    ok = false;
                    break;
                }
                const uint8_t *raw = smem + L.raw + (size_t)slot * L.raw_stage;
                const uint8_t *rawB = raw + L.rawA;
                const float *rawD = reinterpret_cast<const float *>(raw + L.rawA + L.rawB);
                for (int j = 0; j < TC_BPS && ok; ++j, ++blk) {
                    if ((blk & 1) != grp) continue;
                    const int cs = blk % TC_SLOTS, db = blk % TC_BUFS;
                    if (!tc_wait(&tb->op_empty[cs], ((uint32_t)(blk / TC_SLOTS) & 1u) ^ 1u, tb, a.err, lim) ||
                        !tc_wait(&tb->dd_empty[db], ((uint32_t)(blk / TC_BUFS) & 1u) ^ 1u, tb, a.err, lim)) {
                        ok = false;
                        break;
                    }
                    uint8_t *op = smem + L.op + (size_t)cs * TC_OP_BYTES;
#pragma unroll
                    for (int q = 0; q < (2 * TC_M + TC_EXPAND_GROUP - 1) / TC_EXPAND_GROUP; ++q) {
                        const int i = gt + TC_EXPAND_GROUP * q;  // 0..255: A tile i / 128, row i % 128
                        if (i >= 2 * TC_M) break;
                        const int m = i >> 7, r = i & 127;
                        uint4 c0, c1;
                        constexpr int GB = tc_group_bytes(BITS), BPG = GB / (4 * BITS);
                        tc_expand<BITS>(raw + (size_t)m * TC_M * rawrow + (size_t)(j / BPG) * TC_M * GB +
                                            (size_t)r * GB + (j % BPG) * (4 * BITS),
                                        c0, c1);
                        uint8_t *dst = op + m * (TC_M * 32);
                        *reinterpret_cast<uint4 *>(dst + tc_canon(r, 0)) = c0;
                        *reinterpret_cast<uint4 *>(dst + tc_canon(r, 1)) = c1;
                    }
                    if (gt < 2 * TC_N) {
                        const int t = gt >> 1, hf = gt & 1;
                        const uint4 v = *reinterpret_cast<const uint4 *>(rawB + j * (TC_N * 32) + t * 32 + hf * 16);
                        *reinterpret_cast<uint4 *>(op + 2 * TC_M * 32 + tc_canon(t, hf)) = v;
                    }
                    if (gt < TC_N) {
                        double *dd = reinterpret_cast<double *>(smem + L.dd) + db * TC_N;
                        dd[gt] = (double)rawD[gt * TC_BPS + j];
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(&tb->op_full[cs]);
                        mbar_arrive(&tb->dd_full[db]);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&tb->raw_empty[slot]);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        int blk = 0;
        bool ok = true;
        if (lane == 0) {
            for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
                for (int k = 0; k < nblk; ++k, ++blk) {
                    const int cs = blk % TC_SLOTS, bf = blk % TC_BUFS;
                    if (!tc_wait(&tb->op_full[cs], (uint32_t)(blk / TC_SLOTS) & 1u, tb, a.err, lim) ||
                        !tc_wait(&tb->tm_empty[bf], ((uint32_t)(blk / TC_BUFS) & 1u) ^ 1u, tb, a.err, lim)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t op = smem_u32(smem + L.op + (size_t)cs * TC_OP_BYTES);
                    const uint64_t dB = tc_desc(op + 2 * TC_M * 32);
                    tc_mma<BITS>(tmem + (uint32_t)(bf * 64), tc_desc(op), dB);
                    tc_mma<BITS>(tmem + (uint32_t)(bf * 64 + 32), tc_desc(op + TC_M * 32), dB);
                    tc_commit(&tb->op_empty[cs]);
                    tc_commit(&tb->tm_full[bf]);
                }
            }
            // the last MMAs must finish before TMEM is released
            if (blk > 0) {
                const int last = blk - 1;
                mbar_wait(&tb->tm_full[last % TC_BUFS], (uint32_t)(last / TC_BUFS) & 1u, a.err);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        constexpr int NH = TC_N / 2;  // token columns of one warp
        const int e = warp - 4, m = (e >> 2) & 1, hh = e >> 3, q = warp & 3;
        const int c0 = hh * NH;       // first token column
        int blk = 0;
        bool ok = true;
        float *xch = reinterpret_cast<float *>(smem + L.xch) + (size_t)q * TC_N * 32;
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
            int ae, rt, tt;
            decode_item(item, ae, rt, tt);
            const int p0 = a.ws.off[ae] + tt * TC_N;
            const int nt = min(TC_N, a.ws.off[ae + 1] - p0);
            double acc[NH];
#pragma unroll
            for (int t = 0; t < NH; ++t) acc[t] = 0.0;
            for (int k = 0; k < nblk; ++k, ++blk) {
                const int bf = blk % TC_BUFS;
                const uint32_t ph = (uint32_t)(blk / TC_BUFS) & 1u;
                if (!tc_wait(&tb->tm_full[bf], ph, tb, a.err, lim)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t v[NH];
                tc_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(bf * 64 + m * 32 + c0), v);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tb->tm_empty[bf]);
                if (!tc_wait(&tb->dd_full[bf], ph, tb, a.err, lim)) {
                    ok = false;
                    break;
                }
                const double2 *dd = reinterpret_cast<const double2 *>(smem + L.dd) + bf * (TC_N / 2) + c0 / 2;
#pragma unroll
                for (int t = 0; t < NH; t += 2) {
                    const double2 d2 = dd[t >> 1];
                    acc[t] = fma((double)(int)v[t], d2.x, acc[t]);
                    acc[t + 1] = fma((double)(int)v[t + 1], d2.y, acc[t + 1]);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&tb->dd_empty[bf]);
            }
            const float *scales;
            int row0, map_unused;
            a_rows(ae, rt, m, scales, row0, map_unused);
            const int r = row0 + 32 * q + lane;
            const double sw = (double)__ldg(scales + r);
            if (BITS != 8) {
#pragma unroll
                for (int t = 0; t < NH; ++t) acc[t] -= (c0 + t < nt) ? __ldg(a.corr + p0 + c0 + t) : 0.0;
            }
            if (a.down) {
                if (!ok) break;
#pragma unroll
                for (int t = 0; t < NH; ++t)
                    if (c0 + t < nt) a.e_pairs[(size_t)(p0 + c0 + t) * a.H + r] = (float)(acc[t] * sw);
            } else {
                // g and u of this quarter through shared memory (each warp its
                // 16 columns); the gate warp of a half then finishes those
                // columns.  Both warps of a pair pass both barriers even after
                // an abort, so that neither waits for the other forever.
                float *xg = xch + 4 * TC_N * 32;
                if (ok) {
                    float *dst = m ? xch : xg;
#pragma unroll
                    for (int t = 0; t < NH; ++t) dst[(c0 + t) * 32 + lane] = (float)(acc[t] * sw);
                }
                // the two warps of the pair decide together (either failing
                // ends both, at the same item)
                const int bar_id = 1 + q + 4 * hh, pid = 2 * (q + 4 * hh);
                if (lane == 0) *(volatile int *)&tb->pair_ok[pid + m] = ok ? 1 : 0;
                asm volatile("bar.sync %0, 64;" ::"r"(bar_id) : "memory");
                ok = *(volatile int *)&tb->pair_ok[pid] && *(volatile int *)&tb->pair_ok[pid + 1];
                if (m == 0 && ok) {
                    const int nb = a.I / COLI_QBLK;
                    const int tend = min(c0 + NH, nt);
                    for (int t = c0; t < tend; ++t) {
                        const float g = xg[t * 32 + lane];
                        const float u = xch[t * 32 + lane];
                        const double gd = (double)g;
                        const float h = (float)((gd / (1.0 + exp(-gd))) * (double)u);
                        float dh;
                        const int code = q8_lane(h, dh);
                        const int p = p0 + t;
                        a.hq[(size_t)p * a.I + r] = (int8_t)code;
                        if (lane == 0) a.hd[(size_t)p * nb + (r >> 5)] = dh;
                    }
                }
                asm volatile("bar.sync %0, 64;" ::"r"(bar_id) : "memory");
                if (!ok) break;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TC_TMEM_COLS));
    }
}

}  // namespace coli
