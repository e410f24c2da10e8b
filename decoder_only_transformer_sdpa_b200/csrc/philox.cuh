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
// Optionally the bytes are kept in device memory (mask != NULL): a kernel of
// its own (dropout_mask.cu) draws every keep byte of the tiles the kernels
// visit before the forward runs, and the forward and the backward load them
// instead of drawing them.  Byte (query i, key group g) of head bh sits at
// (bh * mask_ld + i) * mask_ld / 8 + g, with mask_ld the tile-padded length:
// the 16 bytes of one query row against one 128-key tile are contiguous and
// 16-byte aligned.
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
        // One 32 x 32 -> 64-bit product per multiplied word gives both halves.
        const uint64_t m0 = (uint64_t)kM0 * c0;
        const uint64_t m1 = (uint64_t)kM1 * c2;
        const uint32_t n0 = (uint32_t)(m1 >> 32) ^ c1 ^ k0;
        const uint32_t n2 = (uint32_t)(m0 >> 32) ^ c3 ^ k1;
        c0 = n0;
        c1 = (uint32_t)m1;
        c2 = n2;
        c3 = (uint32_t)m0;
        k0 += kW0;
        k1 += kW1;
    }
    return make_uint4(c0, c1, c2, c3);
}

// The eight keep bits (bit e = key 8 g + e) of query i, key group g, head bh.
// The eight 16-bit compares run two per word: with the top bit of each half
// of u set and the top bit of each half of t cleared, the subtraction cannot
// borrow from one half into the other, and the top bit of each half of the
// difference tells whether the low 15 bits of u reach those of t; where the
// top bits of u and t differ, u's top bit decides.  The top bit of each half
// is then the keep bit of its key.  A byte permute collects the top bytes of
// two words (keys 4w .. 4w+3 in the sign bits of bytes 0..3), and one multiply
// by 2^0 + 2^7 + 2^14 + 2^21 moves those four sign bits, without carries, to
// bits 28..31 in key order.
__device__ __forceinline__ uint32_t keep_byte(const DropoutParams &dp, uint32_t i, uint32_t g,
                                              uint32_t bh) {
    const uint4 w = philox4x32_10(i, g, bh, dp.offset, dp.k0, dp.k1);
    const uint32_t tt = dp.thr * 0x10001u;   // t in both halves (0 < t < 65536)
    const uint32_t tl = tt & 0x7FFF7FFFu;
    const uint32_t words[4] = {w.x, w.y, w.z, w.w};
    uint32_t f[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t u = words[k];
        const uint32_t d = (u | 0x80008000u) - tl;
        f[k] = (u & ~tt) | (~(u ^ tt) & d);  // bit 15: key 2k kept, bit 31: key 2k + 1
    }
    const uint32_t a = __byte_perm(f[0], f[1], 0x7531) & 0x80808080u;  // keys 0..3
    const uint32_t b = __byte_perm(f[2], f[3], 0x7531) & 0x80808080u;  // keys 4..7
    return ((a * 0x00204081u) >> 28) | (((b * 0x00204081u) >> 24) & 0xF0u);
}

// The same eight keep bits, one 16-bit compare per key.  The backward kernels
// draw with this form: inlined into their (rarely taken) drawing branch, the
// two-per-word form above measured ~4 us slower per GPT-2-sized layer on their
// kept-mask path, which never runs either.
__device__ __forceinline__ uint32_t keep_byte_lanes(const DropoutParams &dp, uint32_t i, uint32_t g,
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

// The backward holds keep bits by key: within each group of eight lanes (the
// keys 8g .. 8g+7), lane s has in byte r the keep bits of those eight keys
// for query (base + s + 8r).  Returns the lane's own key's bits: bit 8r + s =
// keep bit of query (base + s + 8r) for key 8g + (lane & 7).  That is four
// 8 x 8 bit-matrix transposes across the group at once, done in three
// butterfly stages: exchange with lane ^ d (d = 4, 2, 1) and swap the
// off-diagonal d x d blocks, a rotate by +-d bringing the partner's block
// into place and a bit select keeping the lane's own.
__device__ __forceinline__ uint32_t transpose_keep_bits(uint32_t x, int lane) {
#pragma unroll
    for (int st = 0; st < 3; ++st) {
        const int d = 4 >> st;
        const uint32_t m = st == 0 ? 0x0F0F0F0Fu : (st == 1 ? 0x33333333u : 0x55555555u);
        const uint32_t t = __shfl_xor_sync(0xffffffffu, x, d);
        const bool lo = (lane & d) == 0;
        const uint32_t u = __funnelshift_l(t, t, lo ? d : 32 - d);  // rotate left
        const uint32_t own = lo ? m : ~m;
        x = (x & own) | (u & ~own);
    }
    return x;
}

// Offset of the kept byte of query i, key group g, head bh.
__device__ __forceinline__ size_t mask_at(const DropoutParams &dp, uint32_t bh, uint32_t g, uint32_t i) {
    return ((size_t)bh * dp.mask_ld + i) * (dp.mask_ld >> 3) + g;
}

}  // namespace philox
}  // namespace attn
