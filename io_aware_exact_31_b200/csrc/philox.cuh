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
// the counter-based generator Philox-4x32 (Salmon, Moraes, Dror, Shaw,
// "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11) run for 7 rounds (the
// paper reports Philox-4x32 passing TestU01's Crush batteries from 7 rounds
// on; its default of 10 adds a safety margin):
//     W = Philox(counter = (j / 16, i, bh, offset), key = (seed lo, seed hi))
//     u = byte 2 (j % 2) + (j % 4) / 2 of W[(j % 16) / 4]        (8-bit uniform)
//     z_ij = u < t,  t = floor((1 - p) 2^8 + 1/2),  q = t / 2^8
// so one call serves sixteen consecutive keys of a row, and the backward pass
// regenerates exactly the forward's mask from (seed, offset).  The byte order
// (keys 4w, 4w+1, 4w+2, 4w+3 in bytes 0, 2, 1, 3 of word w) puts a pair of
// keys 2c, 2c + 1 in the low bytes of the two 16-bit halves of a word, so one
// borrow-free subtraction decides both (keep_lanes).
#pragma once

#include <stdint.h>

namespace fa {

constexpr int PHILOX_ROUNDS = 7;

struct DropoutParams {
    uint32_t key[2 * PHILOX_ROUNDS];  // round keys: (k0, k1) + r (W0, W1), r = 0..6
    uint32_t offset;                  // counter word 3
    uint32_t lanes_ref;               // (0x8000 + t - 1) in both 16-bit halves
    float keep_scale;                 // 2^8 / t = 1 / q
};

// Philox-4x32 as the SC'11 paper defines it, PHILOX_ROUNDS rounds: each round
// takes the 64-bit products of counter words 0 and 2 with the multipliers
// M0, M1 and forms (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1,
// lo(M0 c0)); the key of round r is the seed plus r times the Weyl
// increments (precomputed on the host into DropoutParams::key).
__device__ __forceinline__ uint4 philox4x32(const DropoutParams& d, uint32_t c0, uint32_t c1,
                                            uint32_t c2, uint32_t c3) {
    constexpr uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
#pragma unroll
    for (int r = 0; r < PHILOX_ROUNDS; ++r) {
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

// Keep decisions of the two keys whose 8-bit numbers sit in the low bytes of
// the 16-bit halves of v (the high bytes zero): bit 15 is set iff the low half
// keeps its key, bit 31 iff the high half does.  In each lane
// (0x8000 + t - 1) - u lies in [0x7F01, 0x80FF] for u, t - 1 < 2^8, so no
// borrow crosses lanes, and its bit 15 is set iff u <= t - 1.
__device__ __forceinline__ uint32_t keep_lanes(uint32_t v, uint32_t lanes_ref) {
    return (lanes_ref - v) & 0x80008000u;
}

// The decisions of the 16 keys of one call, bit k for key k: in word w the
// even lanes (bytes 0, 2) hold keys 4w, 4w + 1 and the odd lanes (bytes 1, 3)
// keys 4w + 2, 4w + 3.  (The forward applies keep_lanes to the words directly,
// in its exponential loop.)
__device__ __forceinline__ uint32_t keep_bits16(const uint4 w, uint32_t lanes_ref) {
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
    uint32_t b = 0;
#pragma unroll
    for (int x = 0; x < 4; ++x) {
        const uint32_t e = keep_lanes(ww[x] & 0x00FF00FFu, lanes_ref);
        const uint32_t o = keep_lanes((ww[x] >> 8) & 0x00FF00FFu, lanes_ref);
        b |= (((e >> 15) & 1u) | ((e >> 30) & 2u) | ((o >> 13) & 4u) | ((o >> 28) & 8u)) << (4 * x);
    }
    return b;
}

// Keep bits of one key (this lane's) against 64 consecutive queries q0 .. q0+63,
// bit c for query q0 + c, with the sixteen lanes of an aligned half-warp
// holding the sixteen keys of one Philox group (key & 15 == lane & 15).  Each
// lane makes the 4 calls for the queries q0 + 16 m + (lane & 15) -- every call
// yields the decisions of all sixteen keys of the group -- and the half-warp
// exchanges them with fifteen xor shuffles (a 16 x 16 bit transpose per m).
__device__ __forceinline__ unsigned long long keep_bits_key_row(const DropoutParams& d, uint32_t key,
                                                                uint32_t q0, uint32_t bh,
                                                                uint32_t lane) {
    const uint32_t w = lane & 15u;
    // D bit 16 m + k: key k of the group (k = 0..15) against query q0 + 16 m + w.
    unsigned long long D = 0ull;
#pragma unroll
    for (uint32_t m = 0; m < 4; ++m) {
        const uint32_t byk = keep_bits16(philox4x32(d, key >> 4, q0 + 16 * m + w, bh, d.offset),
                                         d.lanes_ref);  // bit k = key k
        D |= static_cast<unsigned long long>(byk) << (16 * m);
    }
    constexpr unsigned long long EVERY16 = 0x0001000100010001ull;
    // Own decisions: key w against queries q0 + 16 m + w.
    unsigned long long M = ((D >> w) & EVERY16) << w;
#pragma unroll
    for (uint32_t k = 1; k < 16; ++k) {
        // Send the partner (lane ^ k) its key's decisions (key w ^ k) for the
        // queries q0 + 16 m + w, packed into 4 bits; receive this key's
        // decisions for the queries q0 + 16 m + (w ^ k).
        const unsigned long long s = (D >> (w ^ k)) & EVERY16;
        const uint32_t packed = static_cast<uint32_t>(s | (s >> 15) | (s >> 30) | (s >> 45)) & 0xFu;
        const uint32_t got = __shfl_xor_sync(0xffffffffu, packed, k);
        const unsigned long long g = (got & 1u) | (static_cast<unsigned long long>((got >> 1) & 1u) << 16) |
                                     (static_cast<unsigned long long>((got >> 2) & 1u) << 32) |
                                     (static_cast<unsigned long long>((got >> 3) & 1u) << 48);
        M |= g << (w ^ k);
    }
    return M;
}

}  // namespace fa
