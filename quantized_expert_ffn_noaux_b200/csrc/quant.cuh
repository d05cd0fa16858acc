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

}  // namespace coli
