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
// borrow-free subtraction decides both (keep_mask16).
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

// Keep masks of the two keys whose 8-bit numbers u sit in the low bytes of
// the 16-bit halves of v (the high bytes zero): 0xFFFF in a half whose key is
// kept, 0 otherwise.  In each half (0x8000 + t - 1) - u lies in
// [0x7F01, 0x80FF] for u, t - 1 < 2^8, so no borrow crosses the halves, and
// its bit 15 -- the sign bit of byte 1, or of byte 3 in the high half -- is
// set iff u <= t - 1.  prmt's sign-replicating selectors (8 + byte index)
// spread those two sign bits over their halves.
__device__ __forceinline__ uint32_t keep_mask16(uint32_t v, uint32_t lanes_ref) {
    uint32_t m;
    asm("prmt.b32 %0, %1, 0, 0xBB99;" : "=r"(m) : "r"(lanes_ref - v));
    return m;
}
// Bytes 0 and 2 (even) or 1 and 3 (odd) of w moved to the low bytes of the
// two 16-bit halves, the high bytes zero (prmt selector 4 picks a zero byte).
__device__ __forceinline__ uint32_t byte_lanes(uint32_t w, bool even) {
    uint32_t r;
    if (even) asm("prmt.b32 %0, %1, 0, 0x4240;" : "=r"(r) : "r"(w));
    else asm("prmt.b32 %0, %1, 0, 0x4341;" : "=r"(r) : "r"(w));
    return r;
}

// The decisions of the 16 keys of one call in one 32-bit word: bit j
// (j = 0..7) for key 2j, bit 16 + j for key 2j + 1.  Term j takes the byte
// pair j % 2 (even: bytes 0, 2; odd: bytes 1, 3) of word j / 2, i.e. keys 2j
// and 2j + 1, whose decisions are bits 15 and 31 of the difference of
// keep_mask16; one shift by 15 - j moves both into place.  As a 4-bit
// position index P (bit j: P = j; bit 16 + j: P = 8 + j) the key is
// 2 (P mod 8) + P / 8.
__device__ __forceinline__ uint32_t keep_row16(const uint4 w, uint32_t lanes_ref) {
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
    uint32_t r = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t dj = lanes_ref - byte_lanes(ww[j / 2], j % 2 == 0);
        r |= (dj >> (15 - j)) & (0x80008000u >> (15 - j));
    }
    return r;
}

// Keep bits of one key (this lane's) against 64 consecutive queries q0 .. q0+63,
// with the sixteen lanes of an aligned half-warp holding the sixteen keys of one
// Philox group (key & 15 == lane & 15).  Lane w makes the 4 calls for queries
// q0 + 16 m + w (m = 0..3); call m yields a 16-key row, rows 2h and 2h + 1
// packed into word h (the odd row 8 bits up).  The half-warp then transposes
// its 16 x 16 bit matrices (rows = lanes, columns = position index P) with a
// four-stage butterfly: at distance s, P bit s moves by 16, 4, 2, 1 bit places
// for s = 8, 4, 2, 1, lanes with bit s clear keep the columns with P bit s clear
// and take their partner's other columns, rotated into place (bits a rotation
// wraps fall under the mask).  Lane w then holds position w, i.e. key
// 2 (w mod 8) + w / 8, and one shuffle gives every lane its own key.
// Result: .x covers q0 .. q0+31, .y q0+32 .. q0+63; query q0 + 32 h + 16 b + x
// (b = 0, 1; x = 0..15) is bit (x mod 8) + 16 (x / 8) + 8 b of word h
// (keep_bit_index).
__device__ __forceinline__ uint2 keep_bits_key_row(const DropoutParams& d, uint32_t key, uint32_t q0,
                                                   uint32_t bh, uint32_t lane) {
    const uint32_t w = lane & 15u;
    uint32_t row[4];
#pragma unroll
    for (uint32_t m = 0; m < 4; ++m)
        row[m] = keep_row16(philox4x32(d, key >> 4, q0 + 16 * m + w, bh, d.offset), d.lanes_ref);
    uint32_t a = row[0] | (row[1] << 8), b = row[2] | (row[3] << 8);
    constexpr uint32_t DIST[4] = {8, 4, 2, 1}, SHIFT[4] = {16, 4, 2, 1};
    constexpr uint32_t LOW[4] = {0x0000FFFFu, 0x0F0F0F0Fu, 0x33333333u, 0x55555555u};
#pragma unroll
    for (int st = 0; st < 4; ++st) {
        const bool up = (w & DIST[st]) != 0;
        const uint32_t keep = up ? ~LOW[st] : LOW[st];
        const uint32_t rot = up ? 32u - SHIFT[st] : SHIFT[st];  // rotate left
        const uint32_t pa = __shfl_xor_sync(0xffffffffu, a, DIST[st]);
        const uint32_t pb = __shfl_xor_sync(0xffffffffu, b, DIST[st]);
        a = (a & keep) | (__funnelshift_l(pa, pa, rot) & ~keep);
        b = (b & keep) | (__funnelshift_l(pb, pb, rot) & ~keep);
    }
    const uint32_t src = (lane & 16u) | (w >> 1) | ((w & 1u) << 3);
    a = __shfl_sync(0xffffffffu, a, src);
    b = __shfl_sync(0xffffffffu, b, src);
    return make_uint2(a, b);
}

// Bit of query offset c (0..63) in keep_bits_key_row's word c / 32.
__host__ __device__ constexpr int keep_bit_index(int c) {
    return (c & 7) + 16 * ((c >> 3) & 1) + 8 * ((c >> 4) & 1);
}

}  // namespace fa
