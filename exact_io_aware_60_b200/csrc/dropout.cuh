// dropout.cuh -- the counter-based dropout mask, regenerated wherever it is needed.
//
// Dropout acts on the normalised probabilities between the softmax and the product with
// V (promptingindex page, "Why attention is memory-bound, not compute-bound", where the
// op chain is listed).  Storing an N x N mask would bring back the quadratic memory the
// method removes, so the forward and the backward kernel both recompute it from a
// counter-based generator -- the recomputation principle of the method (anthology note
// "NOTE-005: FlashAttention", "Method") applied to the random numbers.
//
// Generator: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As
// Easy as 1, 2, 3", SC 2011).  Element (i, j) of head bh is decided by byte j mod 16 of
// the 16 output bytes for counter (j / 16, i, bh, offset) and key (seed low word, seed
// high word), byte b being bits 8 (b mod 4) .. +7 of output word b / 4.  It is kept when
// that byte is >= t (t = drop threshold, drop probability t / 256) and kept values are
// scaled by 256 / (256 - t).
#pragma once

#include <cstdint>

namespace fa {

struct DropoutParams {
    uint32_t add16;     // (0x8000 - t) in both 16-bit halves: bit 15 of byte + add16 = keep
    uint32_t seed_lo;
    uint32_t seed_hi;
    uint32_t offset;
    float keep_scale;   // 256 / (256 - t)
};

// One Philox4x32-10 block: ten rounds of the multiply / xor S-box with the key bumped by
// the two Weyl increments after every round.
__device__ __forceinline__ uint4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                               uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        const uint64_t p0 = (uint64_t)c0 * 0xD2511F53u;
        const uint64_t p1 = (uint64_t)c2 * 0xCD9E8D57u;
        c0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
        c1 = (uint32_t)p1;
        c2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
        c3 = (uint32_t)p0;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return make_uint4(c0, c1, c2, c3);
}

// prmt.b32 in its default mode: selector nibble bit 3 replicates the sign of the chosen
// byte over the destination byte.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Bytes 0 and 2 of w (keys 4k, 4k + 2 of a group) into 16-bit lanes plus add16: bit 15 /
// bit 31 of the result say "keep".  Bytes 1 and 3 likewise.
__device__ __forceinline__ uint32_t keep_even(uint32_t w, uint32_t add16) {
    return prmt(w, 0u, 0x4240u) + add16;
}
__device__ __forceinline__ uint32_t keep_odd(uint32_t w, uint32_t add16) {
    return prmt(w, 0u, 0x4341u) + add16;
}

// 16-bit-pair masks for the packed probabilities of keys (4k, 4k+1) and (4k+2, 4k+3) of
// one output word: 0xFFFF where kept, 0 where dropped.
__device__ __forceinline__ void pair_masks(uint32_t w, uint32_t add16, uint32_t &m01,
                                           uint32_t &m23) {
    const uint32_t e = keep_even(w, add16);
    const uint32_t o = keep_odd(w, add16);
    m01 = prmt(e, o, 0xDD99u);
    m23 = prmt(e, o, 0xFFBBu);
}

// The 16 keep bits of one Philox block (bit b = key 16 g + b).
__device__ __forceinline__ uint32_t keep_bits16(uint4 r, uint32_t add16) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
    uint32_t bits = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        // sign bits of bytes 1, 5, 3, 7 of (e, o) = keys 4k, 4k+1, 4k+2, 4k+3
        const uint32_t z = prmt(keep_even(w[k], add16), keep_odd(w[k], add16), 0x7351u);
        // gather the four byte sign bits (7, 15, 23, 31) into bits 28..31
        const uint32_t nib = ((z & 0x80808080u) * 0x00204081u) >> 28;
        bits |= nib << (4 * k);
    }
    return bits;
}

// Transpose, inside each half-warp, the 16 x 16 bit matrices held in the low and the high
// 16 bits of x (lane r of the half holds row r, bit c = column c): afterwards lane c holds
// column c.  Four butterfly stages exchange the off-diagonal quadrants.
__device__ __forceinline__ uint32_t transpose16x16_halfwarp(uint32_t x, int lane) {
#pragma unroll
    for (int j = 8; j >= 1; j >>= 1) {
        const uint32_t m0 = j == 8 ? 0x00FF00FFu : j == 4 ? 0x0F0F0F0Fu : j == 2 ? 0x33333333u
                                                                                    : 0x55555555u;
        const uint32_t y = __shfl_xor_sync(0xffffffffu, x, j);
        x = (lane & j) ? ((x & ~m0) | ((y >> j) & m0)) : ((x & m0) | ((y << j) & ~m0));
    }
    return x;
}

// Writes the keep mask of query rows [0, N) against keys [0, N) of every head:
// keep[bh][i][j] = 1 or 0.  One thread per (bh, i, 16-key group).
__global__ void __launch_bounds__(256) dropout_mask_kernel(uint8_t *keep, long long BH, int N,
                                                          const DropoutParams dp) {
    const int groups = (N + 15) / 16;
    const long long total = BH * (long long)N * groups;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long id = (long long)blockIdx.x * blockDim.x + threadIdx.x; id < total; id += stride) {
        const int g = (int)(id % groups);
        const long long row = id / groups;  // bh * N + i
        const int i = (int)(row % N);
        const uint32_t bh = (uint32_t)(row / N);
        const uint4 r = philox4x32_10((uint32_t)g, (uint32_t)i, bh, dp.offset, dp.seed_lo, dp.seed_hi);
        const uint32_t bits = keep_bits16(r, dp.add16);
        uint8_t *out = keep + row * N + (long long)g * 16;
        const int n = min(16, N - g * 16);
        for (int b = 0; b < n; ++b) out[b] = (uint8_t)((bits >> b) & 1u);
    }
}

}  // namespace fa
