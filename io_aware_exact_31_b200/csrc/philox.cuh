// philox.cuh -- the attention-dropout keep mask.
//
// downcodes.com "triton transformer" (usage section) exposes an attention
// dropout option (attn_dropout) without a formula or a random-number
// convention.  This library reads it as inverted dropout on the normalised
// probabilities: each weight is kept with probability q and kept weights are
// divided by q, so the output is unbiased; LSE stays that of the undropped
// scores.
//
// The keep bit z_ij of query i, key j of query head bh = b * H + h comes from
// the counter-based generator Philox-4x32-10 (Salmon, Moraes, Dror, Shaw,
// "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11):
//     W = Philox(counter = (j / 8, i, bh, offset), key = (seed lo, seed hi))
//     u = (W[(j % 8) / 2] >> 16 (j % 2)) & 0x7FFF            (15-bit uniform)
//     z_ij = u < t,  t = floor((1 - p) 2^15 + 1/2),  q = t / 2^15
// so one call serves eight consecutive keys of a row (two per 32-bit word,
// one per 16-bit half), and the backward pass regenerates exactly the
// forward's mask from (seed, offset).  With 15-bit numbers in 16-bit lanes
// both halves of a word are compared with one borrow-free subtraction.
#pragma once

#include <stdint.h>

namespace fa {

struct DropoutParams {
    uint32_t key[20];     // Philox round keys: (k0, k1) + r (W0, W1), r = 0..9
    uint32_t offset;      // counter word 3
    uint32_t lanes_ref;   // ((t - 1) | 0x8000) in both 16-bit halves
    float keep_scale;     // 2^15 / t = 1 / q
};

// Philox-4x32 with ten rounds, as the SC'11 paper defines it: each round takes
// the 64-bit products of counter words 0 and 2 with the multipliers M0, M1 and
// forms (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1, lo(M0 c0)); the
// key of round r is the seed plus r times the Weyl increments (precomputed on
// the host into DropoutParams::key).
__device__ __forceinline__ uint4 philox4x32_10(const DropoutParams& d, uint32_t c0, uint32_t c1,
                                               uint32_t c2, uint32_t c3) {
    constexpr uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const unsigned long long p0 = static_cast<unsigned long long>(M0) * c0;
        const unsigned long long p1 = static_cast<unsigned long long>(M1) * c2;
        const uint32_t n0 = static_cast<uint32_t>(p1 >> 32) ^ c1 ^ d.key[2 * r];
        const uint32_t n2 = static_cast<uint32_t>(p0 >> 32) ^ c3 ^ d.key[2 * r + 1];
        c1 = static_cast<uint32_t>(p1);
        c3 = static_cast<uint32_t>(p0);
        c0 = n0;
        c2 = n2;
    }
    return make_uint4(c0, c1, c2, c3);
}

// Keep decisions of both 16-bit halves of one output word: bit 15 is set iff
// the low half keeps its key, bit 31 iff the high half does.  In each lane
// (0x8000 + t - 1) - u lies in [1, 0xFFFE] for u, t - 1 < 2^15, so no borrow
// crosses lanes, and its bit 15 is set iff u <= t - 1.
__device__ __forceinline__ uint32_t keep_pair_bits(uint32_t w, uint32_t lanes_ref) {
    return (lanes_ref - (w & 0x7FFF7FFFu)) & 0x80008000u;
}

// Keep bits of query i for the 128 keys [j0, j0 + 128) (j0 a multiple of
// 128): bit 16 e + 4 k + x of keep[c] for key j0 + 32 c + 8 k + 2 x + e.
__device__ __forceinline__ void keep_bits_row128(const DropoutParams& d, uint32_t j0, uint32_t i,
                                                 uint32_t bh, uint32_t (&keep)[4]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) keep[c] = 0;
#pragma unroll 1
    for (int k = 0; k < 4; ++k) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint4 w = philox4x32_10(d, (j0 >> 3) + 4 * c + k, i, bh, d.offset);
            const uint32_t b = (keep_pair_bits(w.x, d.lanes_ref) >> 15) |
                               (keep_pair_bits(w.y, d.lanes_ref) >> 14) |
                               (keep_pair_bits(w.z, d.lanes_ref) >> 13) |
                               (keep_pair_bits(w.w, d.lanes_ref) >> 12);
            keep[c] |= b << (4 * k);
        }
    }
}

// Spread the 8 low bits of x eight apart: bit m goes to bit 8m.
__device__ __forceinline__ unsigned long long spread8(uint32_t x) {
    unsigned long long v = x & 0xFFu;
    v = (v | (v << 28)) & 0x0000000F0000000Full;
    v = (v | (v << 14)) & 0x0003000300030003ull;
    v = (v | (v << 7)) & 0x0101010101010101ull;
    return v;
}

// Keep bits of one key (this lane's) against 64 consecutive queries q0 .. q0+63,
// bit c for query q0 + c, with the eight lanes of an aligned lane octet
// holding the eight keys of one Philox group (key & 7 == lane & 7).  Each lane
// makes the 8 calls for the queries q0 + 8m + (lane & 7) -- every call yields
// the decisions of all eight keys of the group -- and the octet exchanges them
// with seven xor shuffles (an 8 x 8 transpose of bytes).
__device__ __forceinline__ unsigned long long keep_bits_key_row(const DropoutParams& d, uint32_t key,
                                                                uint32_t q0, uint32_t bh,
                                                                uint32_t lane) {
    const uint32_t w = lane & 7u;
    // a[x] bit m (low half) and bit 16 + m (high half): keys 2x and 2x + 1 of
    // the group against query q0 + 8m + w.
    uint32_t a[4] = {0u, 0u, 0u, 0u};
#pragma unroll 2
    for (uint32_t m = 0; m < 8; ++m) {
        const uint4 v = philox4x32_10(d, key >> 3, q0 + 8 * m + w, bh, d.offset);
        a[0] |= keep_pair_bits(v.x, d.lanes_ref) >> (15 - m);
        a[1] |= keep_pair_bits(v.y, d.lanes_ref) >> (15 - m);
        a[2] |= keep_pair_bits(v.z, d.lanes_ref) >> (15 - m);
        a[3] |= keep_pair_bits(v.w, d.lanes_ref) >> (15 - m);
    }
    // Decisions of key x of the group (8 bits, bit m), x = 0..7.
    auto pick = [&](uint32_t x) {
        const uint32_t hi2 = x >> 1;
        const uint32_t r = (hi2 == 0) ? a[0] : (hi2 == 1) ? a[1] : (hi2 == 2) ? a[2] : a[3];
        return (r >> (16 * (x & 1u))) & 0xFFu;
    };
    unsigned long long M = spread8(pick(w)) << w;
#pragma unroll
    for (uint32_t k = 1; k < 8; ++k) {
        // The partner lane ^ k sends its decisions for key w (= its (lane & 7) ^ k);
        // they cover the queries q0 + 8m + (w ^ k).
        const uint32_t got = __shfl_xor_sync(0xffffffffu, pick(w ^ k), k);
        M |= spread8(got) << (w ^ k);
    }
    return M;
}

}  // namespace fa
