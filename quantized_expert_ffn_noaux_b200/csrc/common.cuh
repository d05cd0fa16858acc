// common.cuh -- device helpers shared by the library's kernels (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#define COLI_QBLK 32

namespace coli {

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Q8_0 of one 32-element block held one element per lane:
// d = amax/127 (IEEE fp32 division), q = clamp(rint(x/d), -127, 127).
__device__ __forceinline__ int q8_lane(float x, float &d_out) {
    float amax = warp_max(fabsf(x));
    float d = __fdiv_rn(amax, 127.0f);
    d_out = d;
    float v = 0.0f;
    if (d != 0.0f) v = rintf(__fdiv_rn(x, d));
    v = fminf(fmaxf(v, -127.0f), 127.0f);
    return (int)v;
}

// dp4a with four unsigned 8-bit fields in a and four signed in b.
__device__ __forceinline__ int dp4a_us(unsigned a, int b, int c) {
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ int dp4a_ss(int a, int b, int c) {
    int d;
    asm("dp4a.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ uint4 ldg_stream(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// 16-byte shared-memory load through a 32-bit shared address (volatile, so
// it stays ordered after the mbarrier wait that made the data visible).
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

// ---------------------------------------------------------------------------
// Activation staging.  A weight row of K elements is read as V = K*BITS/128
// uint4 vectors.  For vector v the activation codes it multiplies are stored
// in shared memory as P = 4/ (BITS/2) ... planes of 16 bytes, arranged so the
// unpacked weight fields line up with dp4a operands:
//   BITS 8: plane 0 holds x[16v .. 16v+15] in natural order          (P = 1)
//   BITS 4: vector v is block v; weight word i (elements 8i..8i+7 of the
//           block) unpacks into low nibbles (elements 8i+0,2,4,6) and high
//           nibbles (8i+1,3,5,7); the activation words are stored
//           [E0 O0 E1 O1] in plane 0 and [E2 O2 E3 O3] in plane 1        (P = 2)
//   BITS 2: vector v covers blocks 2v, 2v+1; weight word i holds elements
//           16i + 4j + f in byte j, bits 2f..2f+1; plane i stores the four
//           words G_f = (x[16i+f], x[16i+4+f], x[16i+8+f], x[16i+12+f])  (P = 4)
// Plane p of a row of V vectors starts at p*V*16 bytes.
template <int BITS> struct Fmt {
    static constexpr int ELEMS = 128 / BITS;       // elements per uint4 of weights
    static constexpr int PLANES = ELEMS / 16;      // 16-byte activation planes per uint4
    static constexpr int OFFSET = BITS == 8 ? 0 : (BITS == 4 ? 8 : 2);  // unsigned bias
};

// Byte (element index within the vector's ELEMS) that activation byte
// `pos` (0 .. ELEMS-1, plane-major) must hold.
template <int BITS> __device__ __forceinline__ int stage_src(int pos) {
    if (BITS == 8) return pos;
    if (BITS == 4) {
        int plane = pos >> 4, w = (pos >> 2) & 3, byte = pos & 3;
        int word = plane * 2 + (w >> 1);  // weight word 0..3
        int odd = w & 1;
        return word * 8 + byte * 2 + odd;
    }
    // BITS == 2
    int word = pos >> 4, f = (pos >> 2) & 3, byte = pos & 3;
    return word * 16 + byte * 4 + f;
}

// Raw dp4a sums of one 16-byte weight vector with its activation words.
// Nibbles / crumbs are read as unsigned fields u = code XOR 8 (int4) or
// code XOR 2 (int2), i.e. code + 8 / code + 2; the caller subtracts
// 8 (2) * (sum of the block's activation codes).  (x & m) ^ c compiles to one
// LOP3 per field word.
__device__ __forceinline__ int dot_byte(const uint4 w, const uint4 a) {
    int s = dp4a_ss((int)w.x, (int)a.x, 0);
    s = dp4a_ss((int)w.y, (int)a.y, s);
    s = dp4a_ss((int)w.z, (int)a.z, s);
    return dp4a_ss((int)w.w, (int)a.w, s);
}
__device__ __forceinline__ int dot_nib(const uint4 w, const uint4 a0, const uint4 a1) {
    const unsigned M = 0x0F0F0F0Fu, C = 0x08080808u;
    int s = dp4a_us((w.x & M) ^ C, (int)a0.x, 0);
    s = dp4a_us(((w.x >> 4) & M) ^ C, (int)a0.y, s);
    s = dp4a_us((w.y & M) ^ C, (int)a0.z, s);
    s = dp4a_us(((w.y >> 4) & M) ^ C, (int)a0.w, s);
    s = dp4a_us((w.z & M) ^ C, (int)a1.x, s);
    s = dp4a_us(((w.z >> 4) & M) ^ C, (int)a1.y, s);
    s = dp4a_us((w.w & M) ^ C, (int)a1.z, s);
    return dp4a_us(((w.w >> 4) & M) ^ C, (int)a1.w, s);
}
__device__ __forceinline__ int dot_crumb2(unsigned w0, unsigned w1, const uint4 a0, const uint4 a1) {
    const unsigned M = 0x03030303u, C = 0x02020202u;
    int s = dp4a_us((w0 & M) ^ C, (int)a0.x, 0);
    s = dp4a_us(((w0 >> 2) & M) ^ C, (int)a0.y, s);
    s = dp4a_us(((w0 >> 4) & M) ^ C, (int)a0.z, s);
    s = dp4a_us(((w0 >> 6) & M) ^ C, (int)a0.w, s);
    s = dp4a_us((w1 & M) ^ C, (int)a1.x, s);
    s = dp4a_us(((w1 >> 2) & M) ^ C, (int)a1.y, s);
    s = dp4a_us(((w1 >> 4) & M) ^ C, (int)a1.z, s);
    return dp4a_us(((w1 >> 6) & M) ^ C, (int)a1.w, s);
}

// Sum over the 32 lanes of U per-lane values at once (U a power of two up to
// 16): after the call the total of value r is in every lane with
// lane >> (5 - log2 U) == r (lane >> 4 for U = 2, lane >> 3 for U = 4,
// lane >> 2 for U = 8, lane >> 1 for U = 16).  Exchanging halves first costs
// U - 1 + 5 - log2(U) shuffles instead of 5 U, on a chain 5 steps long.
template <int U>
__device__ __forceinline__ double warp_sum_rows(const double (&v)[U]) {
    static_assert(U == 1 || U == 2 || U == 4 || U == 8 || U == 16, "U: power of two <= 16");
    const int lane = threadIdx.x & 31;
    double cur[U];
#pragma unroll
    for (int i = 0; i < U; ++i) cur[i] = v[i];
    // halving steps: lanes with the offset bit set keep the upper half of
    // the values still in play and send the lower half, the others the
    // reverse; after log2(U) steps value (lane >> (5 - log2 U)) is left
#pragma unroll
    for (int n = U, o = 16; n > 1; n >>= 1, o >>= 1) {
        const bool hi = lane & o;
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
            const double keep = hi ? cur[n / 2 + i] : cur[i];
            const double give = hi ? cur[i] : cur[n / 2 + i];
            cur[i] = keep + __shfl_xor_sync(0xffffffffu, give, o);
        }
    }
    double r = cur[0];
#pragma unroll
    for (int o = 32 / U / 2; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
    return r;
}

// Integer partial dot of one weight vector with its staged activations.
// Returns the raw dp4a sums for each 32-block fragment the vector covers
// (one for BITS 8 -- half a block -- and 4, two for BITS 2), before the
// unsigned-offset correction.
template <int BITS>
__device__ __forceinline__ void vec_dot(const uint4 w, const uint4 *act, int V, int &s0, int &s1) {
    if (BITS == 8) {
        s0 = dot_byte(w, act[0]);
        s1 = 0;
    } else if (BITS == 4) {
        uint4 a0 = act[0], a1 = act[V];
        s0 = dot_nib(w, a0, a1);
        s1 = 0;
    } else {
        uint4 a0 = act[0], a1 = act[V], a2 = act[2 * V], a3 = act[3 * V];
        s0 = dot_crumb2(w.x, w.y, a0, a1);
        s1 = dot_crumb2(w.z, w.w, a2, a3);
    }
}

// fp64 promotion of vector v's partial sums: acc += sum_frag S_frag * d_block.
// xs[b] is the sum of the activation codes of block b (for the offset
// correction), xd[b] its Q8_0 scale.
template <int BITS>
__device__ __forceinline__ double vec_promote(int v, int s0, int s1, const int *xs,
                                              const float *xd, double acc) {
    if (BITS == 8) {
        acc = fma((double)s0, (double)xd[v >> 1], acc);
    } else if (BITS == 4) {
        int S = s0 - 8 * xs[v];
        acc = fma((double)S, (double)xd[v], acc);
    } else {
        int S0 = s0 - 2 * xs[2 * v], S1 = s1 - 2 * xs[2 * v + 1];
        acc = fma((double)S0, (double)xd[2 * v], acc);
        acc = fma((double)S1, (double)xd[2 * v + 1], acc);
    }
    return acc;
}

// Block sums of the vector's fragments after the offset correction
// (exact int32; used by the parity export).
template <int BITS>
__device__ __forceinline__ void vec_block_sums(int v, int s0, int s1, const int *xs, int &b0,
                                               int &S0, int &b1, int &S1) {
    if (BITS == 8) {
        b0 = v >> 1; S0 = s0; b1 = -1; S1 = 0;
    } else if (BITS == 4) {
        b0 = v; S0 = s0 - 8 * xs[v]; b1 = -1; S1 = 0;
    } else {
        b0 = 2 * v; S0 = s0 - 2 * xs[2 * v];
        b1 = 2 * v + 1; S1 = s1 - 2 * xs[2 * v + 1];
    }
}

}  // namespace coli

// ---------------------------------------------------------------------------
// Asynchronous bulk copies (cp.async.bulk, the non-tensor TMA path) into
// shared memory, completed on mbarriers; every wait is bounded.
namespace coli {

// A wait that has not completed after this many SM cycles (~1 s) gives up:
// the kernel records COLI_ETIMEOUT (5) in its error word and returns.
constexpr long long WAIT_LIMIT_CYCLES = 2000000000LL;
constexpr int ERR_TIMEOUT = 5;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking probe of the phase with the given parity.
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait that yields the issue slots while it waits: for threads whose
// wait is long and whose wake-up latency matters little (the producer thread
// waiting for a free ring slot, the epilogue warp waiting for partials), so
// that they do not steal issue cycles from the compute warps of their SM
// sub-partition.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_sleepy(uint64_t *bar, uint32_t parity, int *err,
                                                 long long lim = WAIT_LIMIT_CYCLES) {
    if (mbar_try_wait_hint(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait_hint(bar, parity)) {
        if (clock64() - t0 > lim) {
            if (err) atomicExch(err, ERR_TIMEOUT);
            return false;
        }
        __nanosleep(100);
    }
    return true;
}

// Bounded wait for the phase with the given parity; false (and the error
// word set) if it did not complete within `lim` SM cycles.  Waits for work
// that is sure to finish (copies or MMAs already issued) keep the default
// limit; waits on progress elsewhere may take a shorter per-handle limit.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int *err,
                                          long long lim = WAIT_LIMIT_CYCLES) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > lim) {
            if (err) atomicExch(err, ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

// Global -> shared bulk copy of `bytes` (multiple of 16, both addresses
// 16-byte aligned), completing transaction bytes on `bar`.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// L2 policy for data read once per launch (streamed weights): evict first,
// so that the stream does not push the kernel's code, the routing tables and
// the activation records out of L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ void bulk_g2s_hint(void *dst, const void *src, uint32_t bytes,
                                              uint64_t *bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;"
        ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Release-ordered add at GPU scope: this thread's earlier writes (and those
// ordered before them, e.g. by a warp barrier) are visible to any thread that
// acquires the counter value this add produces.
__device__ __forceinline__ void red_release_add(int *p, int v) {
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Arrive on `bar` once every cp.async this thread issued so far has landed;
// the barrier's expected count includes these arrivals (.noinc).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// Programmatic dependent launch: wait for the preceding grid's completion and
// memory flush; allow the next grid to start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Named barrier among `nthreads` threads (a multiple of 32), id 1..15.  The
// warp reconverges first: bar.sync needs every thread of a warp to arrive at
// the same instruction.
__device__ __forceinline__ void named_bar(int id, int nthreads) {
    __syncwarp();
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------
// Activation records.  One Q8_0 row of length K prepared for a weight format:
//   [0, K)            codes in the staged plane layout of Fmt<BITS>
//   [K, K + 4nb)      int32 sums of the codes of each 32-block
//   [K + 4nb, K + 8nb) fp32 Q8_0 scales
// padded to a multiple of 16 bytes.
__host__ __device__ inline int rec_bytes(int K) {
    return ((K + 8 * (K / COLI_QBLK)) + 15) & ~15;
}

// Byte offset inside the record's code area and the element (0..31 within
// block b) that lane position i of block b holds, for a row of V vectors.
template <int BITS>
__device__ __forceinline__ void rec_slot(int b, int i, int V, int &offset, int &src) {
    if (BITS == 8) {
        const int v = 2 * b + (i >> 4);
        offset = v * 16 + (i & 15);
        src = i;
    } else if (BITS == 4) {
        const int v = b, P = i;
        offset = (P >> 4) * V * 16 + v * 16 + (P & 15);
        src = stage_src<4>(P);
    } else {
        const int v = b >> 1, h = b & 1, P = 32 * h + i;
        offset = (P >> 4) * V * 16 + v * 16 + (P & 15);
        src = stage_src<2>(P) - 32 * h;
    }
}

// Q8_0 of one 32-block held one element per lane, written into a record:
// codes at their staged positions, the block's code sum and scale.
// Optionally also the natural-order codes and scale (q_nat, d_nat).
template <int BITS>
__device__ __forceinline__ void q8_block_to_record(float x, int b, int K, uint8_t *rec,
                                                   int8_t *q_nat, float *d_nat) {
    const int lane = threadIdx.x & 31;
    float d;
    const int code = q8_lane(x, d);
    const int sum = warp_sum_i(code);
    const int V = K * BITS / 128;
    int off, src;
    rec_slot<BITS>(b, lane, V, off, src);
    const int mine = __shfl_sync(0xffffffffu, code, src);
    rec[off] = (uint8_t)(int8_t)mine;
    if (lane == 0) {
        const int nb = K / COLI_QBLK;
        reinterpret_cast<int *>(rec + K)[b] = sum;
        reinterpret_cast<float *>(rec + K + 4 * nb)[b] = d;
    }
    if (q_nat) q_nat[b * COLI_QBLK + lane] = (int8_t)code;
    if (d_nat && lane == 0) d_nat[b] = d;
}

}  // namespace coli
