// philox.cuh -- the attention-dropout keep mask.
//
// downcodes.com "triton transformer" (usage section) exposes an attention
// dropout option (attn_dropout) without a formula or a random-number
// convention.  This library reads it as inverted dropout on the normalised
// probabilities: query i keeps key j with probability 1 - p, kept weights are
// multiplied by 1 / (1 - p), and LSE stays that of the undropped scores.
//
// The keep bit z_ij of query i, key j of query head bh = b * H + h comes from
// the counter-based generator Philox-4x32-10 (Salmon, Moraes, Dror, Shaw,
// "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11):
//     out = Philox(counter = (j / 4, i, bh, offset), key = (seed lo, seed hi))
//     z_ij = out[j % 4] < floor((1 - p) * 2^32)
// so one call serves four consecutive keys of a row, and the backward pass
// regenerates exactly the forward's mask from (seed, offset).
#pragma once

#include <stdint.h>

namespace fa {

struct DropoutParams {
    uint32_t seed_lo, seed_hi;  // the Philox key
    uint32_t offset;            // counter word 3
    uint32_t threshold;         // keep iff word < threshold
    float keep_scale;           // 1 / (1 - p)
};

// Philox-4x32 with ten rounds, as the SC'11 paper defines it: each round takes
// the 64-bit products of counter words 0 and 2 with the multipliers M0, M1 and
// forms (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1, lo(M0 c0)); the
// key advances by the Weyl increments W0, W1 between rounds.
__device__ __forceinline__ uint4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                               uint32_t k0, uint32_t k1) {
    constexpr uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
    constexpr uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const unsigned long long p0 = static_cast<unsigned long long>(M0) * c0;
        const unsigned long long p1 = static_cast<unsigned long long>(M1) * c2;
        const uint32_t n0 = static_cast<uint32_t>(p1 >> 32) ^ c1 ^ k0;
        const uint32_t n2 = static_cast<uint32_t>(p0 >> 32) ^ c3 ^ k1;
        c1 = static_cast<uint32_t>(p1);
        c3 = static_cast<uint32_t>(p0);
        c0 = n0;
        c2 = n2;
        k0 += W0;
        k1 += W1;
    }
    return make_uint4(c0, c1, c2, c3);
}

// Keep bits of the four keys 4g .. 4g+3 of query i: bit x for key 4g + x.
__device__ __forceinline__ uint32_t keep_nibble(const DropoutParams& d, uint32_t g, uint32_t i,
                                                uint32_t bh) {
    const uint4 w = philox4x32_10(g, i, bh, d.offset, d.seed_lo, d.seed_hi);
    return static_cast<uint32_t>(w.x < d.threshold) | (static_cast<uint32_t>(w.y < d.threshold) << 1) |
           (static_cast<uint32_t>(w.z < d.threshold) << 2) |
           (static_cast<uint32_t>(w.w < d.threshold) << 3);
}

// Spread the 16 low bits of x four apart: bit m goes to bit 4m.
__device__ __forceinline__ unsigned long long spread4(uint32_t x) {
    unsigned long long v = x & 0xFFFFu;
    v = (v | (v << 24)) & 0x000000FF000000FFull;
    v = (v | (v << 12)) & 0x000F000F000F000Full;
    v = (v | (v << 6)) & 0x0303030303030303ull;
    v = (v | (v << 3)) & 0x1111111111111111ull;
    return v;
}

// Keep bits of one key (this lane's) against 64 consecutive queries q0 .. q0+63,
// bit c for query q0 + c, with the four lanes of an aligned lane quad holding
// the four keys of one Philox group (key & 3 == lane & 3).  Each lane makes
// the 16 calls for the queries q0 + 4m + (lane & 3) -- every call yields the
// bits of all four keys of the group -- and the quad exchanges them with three
// xor shuffles (a 4 x 4 transpose of 16-bit words).
__device__ __forceinline__ unsigned long long keep_bits_key_row(const DropoutParams& d, uint32_t key,
                                                                uint32_t q0, uint32_t bh,
                                                                uint32_t lane) {
    const uint32_t w = lane & 3u;
    uint32_t lo = 0, hi = 0;  // R_x (x = key within the group) bit m: lo = R0 | R1 << 16, hi = R2 | R3 << 16
#pragma unroll 4
    for (uint32_t m = 0; m < 16; ++m) {
        const uint32_t n = keep_nibble(d, key >> 2, q0 + 4 * m + w, bh);
        lo |= ((n & 1u) << m) | (((n >> 1) & 1u) << (16 + m));
        hi |= (((n >> 2) & 1u) << m) | (((n >> 3) & 1u) << (16 + m));
    }
    auto pick = [&](uint32_t x) { return ((x & 2u) ? hi : lo) >> (16 * (x & 1u)) & 0xFFFFu; };
    unsigned long long M = spread4(pick(w)) << w;
#pragma unroll
    for (uint32_t k = 1; k < 4; ++k) {
        // The partner lane ^ k sends its bits for key w (= its (lane & 3) ^ k);
        // they cover the queries q0 + 4m + (w ^ k).
        const uint32_t got = __shfl_xor_sync(0xffffffffu, pick(w ^ k), k);
        M |= spread4(got) << (w ^ k);
    }
    return M;
}

}  // namespace fa
