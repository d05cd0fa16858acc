// quant.cuh -- Q8_0 activation quantisation and per-row weight quantisation.
//
// Q8_0: "Show HN: 遅いコンピュータで GLM 5.2 を実行する", section 実装済みの主な機能,
// integer-dot bullet (Q8_0-style int8 activations, blocks of 32, one scale).
// Weights: same section, quantisation bullet (int8 / packed int4 / packed
// int2, per-row scales).
#pragma once
#include "common.cuh"

namespace coli {

// One warp per 32-element block; grid-stride over rows * len/32 blocks.
__global__ void k_quant_q8(const float *__restrict__ x, int64_t nblocks, int8_t *__restrict__ q,
                           float *__restrict__ d) {
    const int lane = threadIdx.x & 31;
    int64_t warp = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t b = warp; b < nblocks; b += nwarps) {
        float v = x[b * COLI_QBLK + lane];
        float db;
        int c = q8_lane(v, db);
        q[b * COLI_QBLK + lane] = (int8_t)c;
        if (lane == 0) d[b] = db;
    }
}

template <int BITS> struct WQ {
    static constexpr float QMAX = BITS == 8 ? 127.0f : (BITS == 4 ? 7.0f : 2.0f);
    static constexpr float LO = BITS == 8 ? -127.0f : (BITS == 4 ? -8.0f : -2.0f);
    static constexpr float HI = BITS == 8 ? 127.0f : (BITS == 4 ? 7.0f : 1.0f);
    static constexpr int PER_WORD = 32 / BITS;  // codes per 32-bit output word
};

// One warp per row: amax over the row, scale = amax / qmax, then each lane
// packs 32-bit words of codes (lowest element in the lowest bits).
template <int BITS>
__global__ void k_quant_weights(const float *__restrict__ w, int64_t rows, int64_t K,
                                uint32_t *__restrict__ codes, float *__restrict__ scales) {
    const int lane = threadIdx.x & 31;
    int64_t warp = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t words = K * BITS / 32;
    for (int64_t r = warp; r < rows; r += nwarps) {
        const float4 *row4 = reinterpret_cast<const float4 *>(w + r * K);
        float amax = 0.0f;
        for (int64_t i = lane; i < K / 4; i += 32) {
            float4 f = __ldg(row4 + i);
            amax = fmaxf(amax, fmaxf(fmaxf(fabsf(f.x), fabsf(f.y)), fmaxf(fabsf(f.z), fabsf(f.w))));
        }
        amax = warp_max(amax);
        const float s = __fdiv_rn(amax, WQ<BITS>::QMAX);
        if (lane == 0) scales[r] = s;
        uint32_t *crow = codes + r * words;
        for (int64_t wi = lane; wi < words; wi += 32) {
            uint32_t word = 0;
            const float *src = w + r * K + wi * WQ<BITS>::PER_WORD;
#pragma unroll
            for (int i = 0; i < WQ<BITS>::PER_WORD; ++i) {
                float v = 0.0f;
                if (s != 0.0f) v = rintf(__fdiv_rn(__ldg(src + i), s));
                v = fminf(fmaxf(v, WQ<BITS>::LO), WQ<BITS>::HI);
                uint32_t field = (uint32_t)(int)v & ((1u << BITS) - 1u);
                word |= field << (BITS * i);
            }
            crow[wi] = word;
        }
    }
}

// ---------------------------------------------------------------------------
// FP8 checkpoint weights -> the per-row formats ("Show HN: 遅いコンピュータで
// GLM 5.2 を実行する", 実装済みの主な機能, offline-converter bullet: FP8 shards
// dequantised with 128 x 128 block scales, then requantised).  FP8 is e4m3
// (no infinities); the block scale multiplies:
//   w[r][k] = fp32( e4m3(code[r][k]) * scale[r / B][k / B] )
// and each row is then quantised exactly as k_quant_weights does.

// Two e4m3 codes (low byte first) -> two fp32 values.  Every e4m3 value is
// exactly an fp16 value, so the hardware conversion to f16 is exact.
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t two) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(two));
    float lo, hi;
    asm("{\n .reg .f16 a, b;\n mov.b32 {a, b}, %2;\n cvt.f32.f16 %0, a;\n cvt.f32.f16 %1, b;\n}\n"
        : "=f"(lo), "=f"(hi)
        : "r"(h2));
    return make_float2(lo, hi);
}

// The 16 dequantised weights of one 16-byte group of codes.
__device__ __forceinline__ void fp8x16_dequant(uint4 c, float sc, float (&v)[16]) {
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 a = e4m3x2_to_float2((uint16_t)(w[i] & 0xFFFFu));
        const float2 b = e4m3x2_to_float2((uint16_t)(w[i] >> 16));
        v[4 * i] = __fmul_rn(a.x, sc);
        v[4 * i + 1] = __fmul_rn(a.y, sc);
        v[4 * i + 2] = __fmul_rn(b.x, sc);
        v[4 * i + 3] = __fmul_rn(b.y, sc);
    }
}

// One warp per row; each lane takes 16-code groups (one block scale each,
// B a multiple of 16): pass 1 the row's amax, pass 2 the codes, packed
// lowest element in the lowest bits (16 * BITS / 8 output bytes a group).
template <int BITS>
__global__ void k_requant_fp8(const uint8_t *__restrict__ w8, const float *__restrict__ bscale,
                              int64_t rows, int64_t K, int64_t B, uint8_t *__restrict__ codes,
                              float *__restrict__ scales) {
    const int lane = threadIdx.x & 31;
    int64_t warp = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t groups = K / 16, kb = (K + B - 1) / B;
    for (int64_t r = warp; r < rows; r += nwarps) {
        const uint4 *row = reinterpret_cast<const uint4 *>(w8 + r * K);
        const float *srow = bscale + (r / B) * kb;
        float amax = 0.0f;
        for (int64_t g = lane; g < groups; g += 32) {
            float v[16];
            fp8x16_dequant(__ldg(row + g), __ldg(srow + (g * 16) / B), v);
#pragma unroll
            for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
        }
        amax = warp_max(amax);
        const float s = __fdiv_rn(amax, WQ<BITS>::QMAX);
        if (lane == 0) scales[r] = s;
        uint8_t *crow = codes + r * (K * BITS / 8);
        for (int64_t g = lane; g < groups; g += 32) {
            float v[16];
            fp8x16_dequant(__ldg(row + g), __ldg(srow + (g * 16) / B), v);
            uint32_t word[BITS / 2];
#pragma unroll
            for (int i = 0; i < BITS / 2; ++i) word[i] = 0;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float q = 0.0f;
                if (s != 0.0f) q = rintf(__fdiv_rn(v[i], s));
                q = fminf(fmaxf(q, WQ<BITS>::LO), WQ<BITS>::HI);
                const uint32_t field = (uint32_t)(int)q & ((1u << BITS) - 1u);
                word[i / WQ<BITS>::PER_WORD] |= field << (BITS * (i % WQ<BITS>::PER_WORD));
            }
            uint32_t *dst = reinterpret_cast<uint32_t *>(crow + g * (2 * BITS));
#pragma unroll
            for (int i = 0; i < BITS / 2; ++i) dst[i] = word[i];
        }
    }
}

}  // namespace coli
