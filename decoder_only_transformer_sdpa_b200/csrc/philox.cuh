// philox.cuh -- the counter-based generator behind attention dropout.
//
// Philox4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel Random Numbers: As
// Easy as 1, 2, 3", SC 2011): a 4-word counter is scrambled by ten rounds; a
// round multiplies words 0 and 2 by two fixed odd constants, and the next state
// is (high(M1 c2) ^ c1 ^ k0, low(M1 c2), high(M0 c0) ^ c3 ^ k1, low(M0 c0)); the
// 2-word key grows by two Weyl increments (the fractional parts of the golden
// ratio and of sqrt(3), times 2^32) between rounds.
//
// Dropout mask of the attention weights: element (i, j) of head bh is kept
// iff 16-bit lane (j mod 8) of philox(counter = (i, j / 8, bh, offset),
// key = seed) is >= the threshold t = round(p * 65536); lane e is bits
// 16 (e mod 2) .. +15 of output word e / 2.  Kept weights are scaled by
// 65536 / (65536 - t).
//
// Optionally the bytes are kept in device memory (mask != NULL): the forward
// stores every keep byte it draws, and the backward loads them instead of
// drawing them again.  Byte (query i, key group g) of head bh sits at
// (bh * mask_ld + i) * mask_ld / 8 + g, with mask_ld the tile-padded length:
// a forward thread stores its row's keep bytes four key groups (one word) at a
// time.
#pragma once

#include <stdint.h>

namespace attn {

struct DropoutParams {
    uint32_t k0, k1;     // key: seed low and high words
    uint32_t thr;        // drop threshold t (0 < t < 65536 when dropout is on)
    uint32_t offset;     // counter word 3
    float keep_scale;    // 65536 / (65536 - t)
    uint32_t mask_ld;    // tile-padded T: bytes per key-group row of the kept mask
    uint8_t *mask;       // the kept keep bytes, or NULL (draw them)
};

namespace philox {

constexpr uint32_t kM0 = 0xD2511F53u;
constexpr uint32_t kM1 = 0xCD9E8D57u;
constexpr uint32_t kW0 = 0x9E3779B9u;
constexpr uint32_t kW1 = 0xBB67AE85u;

__device__ __forceinline__ uint4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                               uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint32_t hi0 = __umulhi(kM0, c0), lo0 = kM0 * c0;
        const uint32_t hi1 = __umulhi(kM1, c2), lo1 = kM1 * c2;
        const uint32_t n0 = hi1 ^ c1 ^ k0;
        const uint32_t n2 = hi0 ^ c3 ^ k1;
        c0 = n0;
        c1 = lo1;
        c2 = n2;
        c3 = lo0;
        k0 += kW0;
        k1 += kW1;
    }
    return make_uint4(c0, c1, c2, c3);
}

// The eight keep bits (bit e = key 8 g + e) of query i, key group g, head bh.
__device__ __forceinline__ uint32_t keep_byte(const DropoutParams &dp, uint32_t i, uint32_t g,
                                              uint32_t bh) {
    const uint4 w = philox4x32_10(i, g, bh, dp.offset, dp.k0, dp.k1);
    const uint32_t words[4] = {w.x, w.y, w.z, w.w};
    uint32_t bits = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const uint32_t u = (words[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
        bits |= (u >= dp.thr ? 1u : 0u) << e;
    }
    return bits;
}

// Offset of the kept byte of query i, key group g, head bh.
__device__ __forceinline__ size_t mask_at(const DropoutParams &dp, uint32_t bh, uint32_t g, uint32_t i) {
    return ((size_t)bh * dp.mask_ld + i) * (dp.mask_ld >> 3) + g;
}

}  // namespace philox
}  // namespace attn
