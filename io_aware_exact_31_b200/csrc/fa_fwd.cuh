// fa_fwd.cuh -- exact attention forward for sm_100a (tcgen05 + TMA + TMEM).
//
// Computes, per head and query row i,
//     O_i   = sum_j softmax_j(scale * <q_i, k_j>) v_j     (keys j > i masked if causal)
//     LSE_i = ln sum_j exp(scale * <q_i, k_j>)
// the standard-attention definition of unite.ai "Flash Attention:
// Revolutionizing Transformer Efficiency", evaluated the IO-aware way the same
// page describes ("Flash Attention algorithm": Q/K/V split into blocks that fit
// in on-chip memory, two nested loops, running max m and running sum l) with
// the merge rule of its "math behind Flash Attention" section applied block by
// block, so the N x N score matrix never reaches HBM.  FlashAttention-2's
// changes (systems-analysis.info "FlashAttention-2 (VI)", technical
// architecture items 1-3) map onto this kernel as: 1) the 1/l normalisation is
// deferred to the epilogue and one LSE per row is kept; 2) a head is split
// over CTAs by query block; 3) warps are specialised so that a softmax row
// lives in one thread and needs no shared-memory exchange.
//
// CTA = 2 query tiles of 128 rows (256 rows) of one (batch, head).
//   warps 0-3  softmax warpgroup for tile 0 (thread = one query row = one TMEM lane)
//   warps 4-7  softmax warpgroup for tile 1
//   warp  8    tcgen05.mma issuer; owns the TMEM allocation
//   warp  9    TMA producer (Q once, then the K/V ring)
//   warps 10-11 idle (they complete the third warpgroup, which setmaxnreg needs);
//              at d = 64 they issue the P.V MMAs of tile 0 and tile 1 (below)
// TMEM (512 columns): S0 [0,128)  S1 [128,256)  O0 [256,256+D)  O1 [256+D,256+2D)
//   P_t (bf16, two per column) overwrites the first 64 columns of S_t and is
//   read by the P.V MMA straight from TMEM.
// Tensor-core issue order per key block j (P aliasing S requires PV_t(j-1)
// before S_t(j); tcgen05 ops of one thread execute in order):
//   PV0(j-1) S0(j) PV1(j-1) S1(j)
// so softmax of tile 0 overlaps the tile-1 GEMMs and vice versa, and the
// commit that publishes S_t(j) also guarantees PV_t(j-1) is complete, which is
// when the softmax warps may rescale O_t in place.
//
// d = 64 (bf16) leaves 128 TMEM columns free, enough for P in columns of its
// own: P0 [384,448)  P1 [448,512).  S_t(j+1) then no longer waits for the
// softmax of block j to finish -- only for its threads to have read S_t(j)
// (barrier s_free) -- so it is computed while the exponentials of block j
// run, and the per-tile chain S -> softmax -> P.V -> S is broken.  Three
// threads issue the MMAs: warp 8 all S_t, warps 10 and 11 the P.V of tile 0
// and tile 1, so that each issuing thread waits only on the barriers of its
// own instructions.  The softmax waits for P.V_t(j-1)
// (barrier pv_done) before it rescales O_t or overwrites P_t.  One tile's S(j)
// waits until the other tile is halfway through its exponentials of block j
// (barrier exp_mark), which keeps the two tiles' exponential phases apart.
#pragma once

#include "philox.cuh"
#include "sm100.cuh"

namespace fa {

constexpr int FWD_BM = 128;          // query rows per tile (= TMEM lanes)
constexpr int FWD_BN = 128;          // keys per block
constexpr int FWD_THREADS = 384;     // 12 warps = 3 warpgroups
// Registers: launched at 168/thread (384 x 168 = 64512); the control
// warpgroup gives back down to 72 and each softmax warpgroup takes 216:
// 2 x 128 x 216 + 128 x 72 = 64512.
constexpr uint32_t FWD_REGS_SOFTMAX = 216;
constexpr uint32_t FWD_REGS_CONTROL = 72;
constexpr float FWD_RESCALE_TAU = 8.0f;  // log2 units: keep a stale row max while p <= 2^8

// F8: Q, K, V and P in E4M3 (kind::f8f6f4 MMAs); otherwise bf16 (kind::f16).
template <int D, bool F8 = false>
struct FwdCfg {
    static constexpr int ESZ = F8 ? 1 : 2;                 // operand bytes per element
    static constexpr int TILE_BYTES = FWD_BM * D * ESZ;    // one Q, K or V tile
    static constexpr int NK = 3;                           // K ring depth
    static constexpr int NV = (D * ESZ == 256) ? 2 : 3;    // V ring depth
    static constexpr int PREFETCH = 2;                     // L2 prefetch distance beyond the rings
    static constexpr int BOX_ELEMS = 128 / ESZ;            // elements per 128-B TMA box row
    static constexpr int CHUNKS = D / BOX_ELEMS;           // TMA boxes per tile
    static constexpr int KSTEP = 32 / ESZ;                 // MMA k per instruction (32 B)
    static constexpr int PV_PER_HALF = 64 / KSTEP;         // P.V instructions per 64 keys
    static constexpr int P_COLS_HALF = 64 * ESZ / 4;       // TMEM columns of 64 keys of P
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + 2 * TILE_BYTES;
    static constexpr int OFF_V = OFF_K + NK * TILE_BYTES;
    static constexpr int OFF_BAR = OFF_V + NV * TILE_BYTES;
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM_BYTES = OFF_BAR + BAR_BYTES + 1024;  // + alignment slack
    static constexpr uint32_t TMEM_S0 = 0, TMEM_S1 = 128, TMEM_O0 = 256, TMEM_O1 = 256 + D;
    // P in its own columns (see the header): d = 64 with bf16 operands.
    static constexpr bool SEP = (D == 64) && !F8;
    static constexpr uint32_t TMEM_P0 = 256 + 2 * D, TMEM_P1 = 256 + 2 * D + 64;
    static_assert(!SEP || TMEM_P1 + 64 <= 512, "P columns exceed TMEM");
};

struct FwdParams {
    __nv_bfloat16* O;
    float* LSE;
    int N;              // sequence length
    int n_kv_blocks;    // ceil(N / 128)
    float scale_log2;   // scale * log2(e) (times the Q and K dequant scales for E4M3)
    float o_scale;      // V dequant scale for E4M3 inputs (1 for bf16)
    int causal;
    int n_heads;        // B * H (query heads)
    int H;              // query heads per batch
    int group;          // query heads per K/V head (H / H_kv; 1 = plain multi-head)
    const int* seqlens; // [B] real tokens per batch (device), or null: all N are real
    int n_pairs;        // ceil(N / 256)
    uint32_t* err;      // device error word
    DropoutParams drop; // attention dropout (kernels instantiated with DROP only)
};

// Barrier slots inside the barrier area.
struct FwdBars {
    uint64_t q_full;
    uint64_t k_full[3], k_empty[3];
    uint64_t v_full[3], v_empty[3];
    uint64_t s_full[2], p_full[2][2], o_full[2];  // p_full[tile][key half]
    uint64_t s_free[2], pv_done[2];               // separate-P layout only
    uint64_t exp_mark;                            // separate-P layout: the leading tile halfway through its exponentials
};
static_assert(sizeof(FwdBars) + 8 <= 256, "barrier area");

// DROP: attention dropout (philox.cuh) on the bf16 path; the 1 / (1 - p)
// factor arrives folded into p.o_scale.
template <int D, bool F8 = false, bool DROP = false>
__global__ void __launch_bounds__(FWD_THREADS, 1)
fa_fwd_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
              const __grid_constant__ CUtensorMap mapV, const __grid_constant__ CUtensorMap mapO,
              const FwdParams p) {
    static_assert(!(F8 && DROP), "dropout is implemented for bf16 operands only");
    using C = FwdCfg<D, F8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    FwdBars* bars = reinterpret_cast<FwdBars*>(smem + C::OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + sizeof(FwdBars));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const Guard g{abort_flag, p.err};

    const uint32_t warp = warp_id(), lane = lane_id();
    // 1-D grid.  Causal: block b -> (pair, head) with the pair index
    // outermost and descending, so every head's heaviest (last) query pairs
    // are dispatched first and the light ones fill the final wave.
    // Non-causal (all CTAs equal): head-major, the pairs of one head adjacent,
    // so the CTAs resident at one time share few heads' K/V in L2.
    int bh, pair;
    if (p.causal) {
        bh = blockIdx.x % p.n_heads;
        pair = p.n_pairs - 1 - static_cast<int>(blockIdx.x / p.n_heads);
    } else {
        bh = blockIdx.x / p.n_pairs;
        pair = blockIdx.x % p.n_pairs;
    }
    // K/V head of this query head (grouped-query attention; = bh when group = 1).
    const int bkv = (bh / p.H) * (p.H / p.group) + (bh % p.H) / p.group;
    const int q0 = pair * 2 * FWD_BM;
    // Padded batches: tokens >= len of this batch are padding -- masked as
    // keys, zero output as queries; key blocks past len are never loaded.
    const int len = p.seqlens ? min(max(__ldg(p.seqlens + bh / p.H), 0), p.N) : p.N;
    const int n_kv = (len + FWD_BN - 1) / FWD_BN;
    const bool padding_cta = q0 >= len;  // all rows of this CTA are padding
    // Key blocks each tile needs: causal tiles stop at their diagonal block.
    int n_tile[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const int last_row = q0 + (t + 1) * FWD_BM - 1;
        n_tile[t] = padding_cta ? 0 : p.causal ? min(last_row / FWD_BN + 1, n_kv) : n_kv;
    }
    const int n_blocks = n_tile[1];  // n_tile[0] <= n_tile[1] <= n_tile[0] + 1
    // d = 64: the tile whose exponentials lead the other's by half a softmax
    // (below).  With causal masking tile 1, which may have the extra block, so
    // that the follower ends about when the leader does; otherwise tile 0
    // (measured: 4x16x2048x64 causal 454 -> 476 TFLOP/s with tile 1 leading,
    // 4x16x4096x64 704 -> 675).
    const int lead = p.causal ? 1 : 0;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        mbar_init(&bars->q_full, 1);
        for (int s = 0; s < C::NK; ++s) {
            mbar_init(&bars->k_full[s], 1);
            mbar_init(&bars->k_empty[s], 1);
        }
        for (int s = 0; s < C::NV; ++s) {
            mbar_init(&bars->v_full[s], 1);
            mbar_init(&bars->v_empty[s], C::SEP ? 2 : 1);  // SEP: one commit per P.V issuer
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bars->s_full[t], 1);
            mbar_init(&bars->p_full[t][0], 128);
            mbar_init(&bars->p_full[t][1], 128);
            mbar_init(&bars->o_full[t], 1);
            mbar_init(&bars->s_free[t], 128);
            mbar_init(&bars->pv_done[t], 1);
            if (t == 0) mbar_init(&bars->exp_mark, 4);
        }
        fence_barrier_init();
    }
    if (warp == 8) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp >= 10) {
        regs_decrease<FWD_REGS_CONTROL>();
        if constexpr (C::SEP) {
            // -------------------------------------------- P.V issuer of tile t
            const int t = static_cast<int>(warp) - 10;
            if (!padding_cta) {  // the whole warp; one elected lane issues
                const uint32_t idO = idesc_bf16(128, D, false, true);
                const uint32_t sV = smem_u32(smem + C::OFF_V);
                const uint32_t tO = tmem + (t == 0 ? C::TMEM_O0 : C::TMEM_O1);
                const uint32_t tP = tmem + (t == 0 ? C::TMEM_P0 : C::TMEM_P1);
                bool ok = true;
                for (int j = 0; ok && j < n_blocks; ++j) {
                    const int sv = j % C::NV;
                    if (!(ok = mbar_wait_warp(&bars->v_full[sv], (j / C::NV) & 1, g, 17 + t))) break;
                    if (j < n_tile[t]) {
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            if (!(ok = mbar_wait_warp(&bars->p_full[t][h], j & 1, g, 19 + 2 * t + h))) break;
                            tc_fence_after();
                            // O_t (+)= P_t V_j for keys [64h, 64h + 64): P from
                            // TMEM (8 columns per instruction), V MN-major.
                            // descriptor of this V stage; k-steps advance its
                            // address field (16-byte units, no carry: < 256 KB)
                            const uint64_t b0 = sdesc_sw128(sV + sv * C::TILE_BYTES, 16384, 1024);
                            const int kk0 = h * C::PV_PER_HALF;
                            mma_ts_blk<C::PV_PER_HALF, 8, C::KSTEP * 8>(
                                tO, tP + kk0 * 8, desc_off(b0, kk0 * C::KSTEP * 8), idO,
                                (j > 0 || h > 0) ? 1u : 0u);
                        }
                        if (!ok) break;
                        tc_commit_w(&bars->pv_done[t]);
                    }
                    // Both issuers release V(j), whether or not this tile used it.
                    tc_commit_w(&bars->v_empty[sv]);
                }
            }
        }
    } else if (warp == 9) {
        regs_decrease<FWD_REGS_CONTROL>();
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && !padding_cta) {
            tma_prefetch_desc(&mapQ);
            tma_prefetch_desc(&mapK);
            tma_prefetch_desc(&mapV);
            mbar_arrive_expect_tx(&bars->q_full, 2 * C::TILE_BYTES);
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int c = 0; c < C::CHUNKS; ++c)
                    tma_load_3d(smem + C::OFF_Q + t * C::TILE_BYTES + c * 16384, &mapQ,
                                &bars->q_full, c * C::BOX_ELEMS, q0 + t * FWD_BM, bh);
            // K(j) and V(j) go to their own rings; L2 is asked for the tiles
            // PREFETCH blocks beyond what the rings hold.
            int k_issued = 0, v_issued = 0;
            for (int j = 0; j < n_blocks; ++j) {
                const int sk = j % C::NK, sv = j % C::NV;
                if (j >= C::NK && !mbar_wait(&bars->k_empty[sk], ((j / C::NK) & 1) ^ 1, g, 1)) break;
                mbar_arrive_expect_tx(&bars->k_full[sk], C::TILE_BYTES);
#pragma unroll
                for (int c = 0; c < C::CHUNKS; ++c)
                    tma_load_3d(smem + C::OFF_K + sk * C::TILE_BYTES + c * 16384, &mapK,
                                &bars->k_full[sk], c * C::BOX_ELEMS, j * FWD_BN, bkv);
                k_issued = j + 1;
                const int jp = j + C::NK + C::PREFETCH - 1;
                if (jp < n_blocks) {
#pragma unroll
                    for (int c = 0; c < C::CHUNKS; ++c) {
                        tma_prefetch_l2_3d(&mapK, c * C::BOX_ELEMS, jp * FWD_BN, bkv);
                        tma_prefetch_l2_3d(&mapV, c * C::BOX_ELEMS, jp * FWD_BN, bkv);
                    }
                }
                if (j >= C::NV && !mbar_wait(&bars->v_empty[sv], ((j / C::NV) & 1) ^ 1, g, 2)) break;
                mbar_arrive_expect_tx(&bars->v_full[sv], C::TILE_BYTES);
#pragma unroll
                for (int c = 0; c < C::CHUNKS; ++c)
                    tma_load_3d(smem + C::OFF_V + sv * C::TILE_BYTES + c * 16384, &mapV,
                                &bars->v_full[sv], c * C::BOX_ELEMS, j * FWD_BN, bkv);
                v_issued = j + 1;
            }
            // Never leave the CTA with copies still landing in its shared
            // memory: wait (bounded) for the last load issued into each slot.
            mbar_drain(&bars->q_full, 0);
            for (int j = max(0, k_issued - C::NK); j < k_issued; ++j)
                mbar_drain(&bars->k_full[j % C::NK], (j / C::NK) & 1);
            for (int j = max(0, v_issued - C::NV); j < v_issued; ++j)
                mbar_drain(&bars->v_full[j % C::NV], (j / C::NV) & 1);
        }
    } else if (warp == 8) {
        // ------------------------------------------------------------ MMA issuer
        regs_decrease<FWD_REGS_CONTROL>();
        if (!padding_cta) {  // the whole warp; one elected lane issues
            // S = Q K^T (K-major A, B); O += P V (V MN-major)
            const uint32_t idS = F8 ? idesc_e4m3(128, FWD_BN, false) : idesc_bf16(128, FWD_BN, false, false);
            const uint32_t idO = F8 ? idesc_e4m3(128, D, true) : idesc_bf16(128, D, false, true);
            const uint32_t sQ = smem_u32(smem + C::OFF_Q);
            const uint32_t sK = smem_u32(smem + C::OFF_K);
            const uint32_t sV = smem_u32(smem + C::OFF_V);
            const uint32_t tS[2] = {tmem + C::TMEM_S0, tmem + C::TMEM_S1};
            const uint32_t tO[2] = {tmem + C::TMEM_O0, tmem + C::TMEM_O1};

            // S_t = Q_t K_j^T : K-major A and B, steps of 32 bytes along d.
            auto issue_S = [&](int t, int s) {
                const uint64_t a0 = sdesc_sw128(sQ + t * C::TILE_BYTES, 16, 1024);
                const uint64_t b0 = sdesc_sw128(sK + s * C::TILE_BYTES, 16, 1024);
                if constexpr (F8)
                    mma_ss_f8_blk<D / C::KSTEP, FA_STEP_KMAJOR, FA_STEP_KMAJOR>(tS[t], a0, b0, idS, 0u);
                else
                    mma_ss_blk<D / C::KSTEP, FA_STEP_KMAJOR, FA_STEP_KMAJOR>(tS[t], a0, b0, idS, 0u);
            };
            // O_t (+)= P_t V_j for keys [64h, 64h + 64): P from TMEM (8 columns
            // per instruction), V MN-major (KSTEP key rows of 128 B per step).
            // The two halves are issued as soon as the softmax warps release
            // each half of P.
            auto issue_PV_half = [&](int t, int s, int h, bool acc) {
                const uint64_t b0 = sdesc_sw128(sV + s * C::TILE_BYTES, 16384, 1024);
                const int kk0 = h * C::PV_PER_HALF;
                const uint64_t b = desc_off(b0, kk0 * C::KSTEP * 8);
                const uint32_t en = (acc || h > 0) ? 1u : 0u;
                if constexpr (F8)
                    mma_ts_f8_blk<C::PV_PER_HALF, 8, C::KSTEP * 8>(tO[t], tS[t] + kk0 * 8, b, idO, en);
                else
                    mma_ts_blk<C::PV_PER_HALF, 8, C::KSTEP * 8>(tO[t], tS[t] + kk0 * 8, b, idO, en);
            };

            bool ok = mbar_wait_warp(&bars->q_full, 0, g, 3);
            if constexpr (C::SEP) {
                // S issuer: S_t(j) as soon as K(j) is in and the softmax threads
                // of tile t have read S_t(j - 1) into registers.
                for (int j = 0; ok && j < n_blocks; ++j) {
                    const int sk = j % C::NK;
                    if (!(ok = mbar_wait_warp(&bars->k_full[sk], (j / C::NK) & 1, g, 5))) break;
#pragma unroll
                    for (int tt = 0; tt < 2; ++tt) {
                        const int t = (tt == 0) ? lead : 1 - lead;
                        if (j < n_tile[t]) {
                            if (j > 0 && !(ok = mbar_wait_warp(&bars->s_free[t], (j - 1) & 1, g, 15 + t)))
                                break;
                            // The follower's S(j) only once the leading tile has
                            // made the first half of its weights of block j
                            // (barrier exp_mark, one arrival per leading warp).
                            // Left alone the two tiles run in lock step, both
                            // warps of a sub-partition in their exponentials at
                            // once and then both idle on the ex2 unit while they
                            // wait for S and load it; held half a softmax apart
                            // every block, each warp's loads and waits fall in
                            // the other's exponentials.
                            if (t != lead && !(ok = mbar_wait_warp(&bars->exp_mark, j & 1, g, 50)))
                                break;
                            tc_fence_after();
                            issue_S(t, sk);
                            tc_commit_w(&bars->s_full[t]);
                        }
                    }
                    if (!ok) break;
                    tc_commit_w(&bars->k_empty[sk]);
                }
            } else {  // P over S: one issuer for every MMA
                ok = ok && mbar_wait_warp(&bars->k_full[0], 0, g, 4);
                if (ok) {
                    tc_fence_after();
                    issue_S(0, 0);
                    tc_commit_w(&bars->s_full[0]);
                    issue_S(1, 0);
                    tc_commit_w(&bars->s_full[1]);
                    tc_commit_w(&bars->k_empty[0]);
                }
                for (int j = 1; ok && j <= n_blocks; ++j) {
                    // Finish block j-1 (P.V) for both tiles, then start block j (S).
                    // Each wait sits right before the first MMA that needs it, and
                    // V(j-1)'s slot is released right after its last P.V.
                    const int sv = (j - 1) % C::NV;
                    const uint32_t phv = ((j - 1) / C::NV) & 1;
                    const int sk = j % C::NK;
                    const uint32_t phk = (j / C::NK) & 1;
                    const bool more = j < n_blocks;
                    bool k_ready = false;
                    if (!(ok = mbar_wait_warp(&bars->v_full[sv], phv, g, 6))) break;
                    tc_fence_after();
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        if (j - 1 < n_tile[t]) {
                            if (!(ok = mbar_wait_warp(&bars->p_full[t][0], (j - 1) & 1, g, 7 + t))) break;
                            tc_fence_after();
                            issue_PV_half(t, sv, 0, j > 1);
                            if (!(ok = mbar_wait_warp(&bars->p_full[t][1], (j - 1) & 1, g, 13 + t))) break;
                            tc_fence_after();
                            issue_PV_half(t, sv, 1, true);
                            if (j == n_tile[t]) tc_commit_w(&bars->o_full[t]);
                        }
                        if (t == 1) tc_commit_w(&bars->v_empty[sv]);
                        if (more && j < n_tile[t]) {
                            if (!k_ready) {
                                if (!(ok = mbar_wait_warp(&bars->k_full[sk], phk, g, 5))) break;
                                tc_fence_after();
                                k_ready = true;
                            }
                            issue_S(t, sk);
                            tc_commit_w(&bars->s_full[t]);
                        }
                    }
                    if (!ok) break;
                    if (more) tc_commit_w(&bars->k_empty[sk]);
                }
            }
        }
    } else {
        // ------------------------------------------------------------ softmax warpgroups
        regs_increase<FWD_REGS_SOFTMAX>();
        const int t = warp / 4;                    // tile
        const uint32_t lane_base = (warp % 4) * 32;  // TMEM lane quarter of this warp
        const int row = lane_base + lane;          // row inside the tile
        const int q = q0 + t * FWD_BM + row;       // query index
        const uint32_t tS = tmem_addr(tmem, lane_base, t == 0 ? C::TMEM_S0 : C::TMEM_S1);
        const uint32_t tO = tmem_addr(tmem, lane_base, t == 0 ? C::TMEM_O0 : C::TMEM_O1);
        // Where P goes: over the first columns of S_t, or its own columns (SEP).
        const uint32_t tP =
            C::SEP ? tmem_addr(tmem, lane_base, t == 0 ? C::TMEM_P0 : C::TMEM_P1) : tS;
        const float sl2 = p.scale_log2;
        float m_used = -INFINITY;  // running row max, log2 units of scaled scores
        float l = 0.f;             // running row sum of exp2(s*sl2 - m_used) (for LSE)
        float lr = 0.f;            // same sum over the bf16-rounded weights (for O)
        bool ok = true;
        const int nt = n_tile[t];
        const int tile_first_q = q0 + t * FWD_BM;
        for (int j = 0; j < nt; ++j) {
            uint4 dw = make_uint4(0u, 0u, 0u, 0u);  // DROP: Philox output of the current 16 keys
            if (!(ok = mbar_wait_warp(&bars->s_full[t], j & 1, g, 9 + t))) break;
            tc_fence_after();
            uint32_t sr[128];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sr + c * 32);
            tmem_ld_wait();
            reg_fence<128>(sr);
            if constexpr (C::SEP) {
                // S_t is in registers: the tensor core may overwrite it with S_t(j+1).
                tc_fence_before();
                mbar_arrive(&bars->s_free[t]);
            }
            float s[128];
#pragma unroll
            for (int i = 0; i < 128; ++i) s[i] = __uint_as_float(sr[i]);
            const int key0 = j * FWD_BN;
            // Mask keys past the end and (causal) keys after the query.
            const bool tail = key0 + FWD_BN > len;
            const bool diag = p.causal && key0 + FWD_BN - 1 > tile_first_q;
            if (tail || diag) {
                const int lim = p.causal ? min(q + 1, len) : len;  // valid keys: key < lim
#pragma unroll
                for (int i = 0; i < 128; ++i)
                    if (key0 + i >= lim) s[i] = -INFINITY;
            }
            // Row max: eight independent three-input chains (short dependency depth).
            auto row_max = [&]() {
                float a[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) a[k] = fmaxf(s[2 * k], s[2 * k + 1]);
#pragma unroll
                for (int i = 16; i < 128; i += 16)
#pragma unroll
                    for (int k = 0; k < 8; ++k) a[k] = fmax3(a[k], s[i + 2 * k], s[i + 2 * k + 1]);
                return fmaxf(fmax3(a[0], a[1], a[2]), fmax3(fmax3(a[3], a[4], a[5]), a[6], a[7]));
            };
            // With P in its own columns (and no dropout, whose kernel would
            // spill with both paths) the blocks after the first skip the row
            // max: their weights are taken against the running reference as it
            // stands, and only a block whose weights reach 2^64 against it
            // (checked on the row sum below) is redone against its own max.
            // O and l stay exact either way (one reference for both); 2^64
            // keeps every fp32 accumulation far from overflow.
            constexpr bool kLazyMax = C::SEP && !DROP;
            const bool lazy_max = kLazyMax && j > 0;
            float alpha = 1.f;
            if (!lazy_max) {
                const float m_blk = row_max() * sl2;
                if (j == 0) {
                    m_used = m_blk;
                } else if (m_blk > m_used + FWD_RESCALE_TAU) {
                    alpha = ex2_approx(m_used - m_blk);
                    m_used = m_blk;
                }
            }
            // A row whose keys are all masked so far keeps m = -inf; use 0 so
            // exp2(-inf - 0) = 0 instead of NaN.
            float m_sub = (m_used == -INFINITY) ? 0.f : m_used;
            // Rescale O_t in place when this row's max moved (rare after the
            // first blocks).  PV_t(j-1) must be complete: with P over S it was
            // issued before S_t(j), whose commit we waited for; with P in its
            // own columns the softmax waits for pv_done first (below).
            auto rescale_O = [&]() {
                if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(tO + c * 32, o);
                        tmem_ld_wait();
                        reg_fence<32>(o);
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                        tmem_st32(tO + c * 32, o);
                    }
                }
            };
            if constexpr (!C::SEP) rescale_O();
            l *= alpha;
            lr *= alpha;
            // p = exp2(s * scale_log2 - m), rounded to bf16 for the P.V product.
            // Two row sums: the exact one (for LSE) and one over the SAME rounded
            // weights the tensor core multiplies V with, used to normalise O, so
            // that O = sum p~ v / sum p~ is an exact convex combination of value
            // rows (a row dominated by one key returns that value row exactly).
            // P goes to TMEM as bf16 pairs (key 2c in the low half of column c),
            // or for E4M3 operands four per column (key 4c + b in byte b).
            // Packed f32x2 arithmetic, four independent accumulators per sum.
            const float2 sl2v = make_float2(sl2, sl2);
            float2 ae[4], ar[4];
            // The weights of keys [64h, 64h + 64) into pk, both row sums into ae / ar.
            auto exp_half = [&](int h, float msub, uint32_t (&pk)[32]) {
                const float2 negm = make_float2(-msub, -msub);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float2 x =
                        __ffma2_rn(make_float2(s[h * 64 + 2 * i], s[h * 64 + 2 * i + 1]), sl2v, negm);
                    const float2 pe = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                    ae[i % 4] = __fadd2_rn(ae[i % 4], pe);
                    if constexpr (F8) {
                        // four E4M3 per column: keys 4c..4c+3 in bytes 0..3
                        const uint32_t h16 = pack_e4m3x2(pe.x, pe.y);
                        if (i & 1) {
                            pk[i / 2] |= h16 << 16;
                            float2 a, b;
                            unpack_e4m3x4(pk[i / 2], a, b);
                            ar[i % 4] = __fadd2_rn(ar[i % 4], __fadd2_rn(a, b));
                        } else {
                            pk[i / 2] = h16;
                        }
                    } else {
                        pk[i] = pack_bf16x2(pe.x, pe.y);
                        add_bf16x2_f32(ar[i % 4], pk[i]);
                        if constexpr (DROP) {
                            // Dropped weights leave the P.V product but stay in
                            // both row sums (the softmax is of undropped scores).
                            // Keys 64h + 2i (low half of pk[i]) and 64h + 2i + 1
                            // (high half): one Philox call per 16 keys, made here
                            // where its integer work overlaps the exponentials;
                            // the pair's bytes sit in the two 16-bit lanes of
                            // word (i % 8) / 2 (bytes 0/2 for even i, 1/3 for odd
                            // i); keep_mask16 turns the two decisions into the
                            // 16-bit masks of the pair.
                            if (i % 8 == 0)
                                dw = philox4x32(p.drop,
                                                static_cast<uint32_t>((j * FWD_BN) / 16 + 4 * h + i / 8),
                                                static_cast<uint32_t>(q), static_cast<uint32_t>(bh),
                                                p.drop.offset);
                            const uint32_t wd = ((i % 8) / 2 == 0)   ? dw.x
                                                : ((i % 8) / 2 == 1) ? dw.y
                                                : ((i % 8) / 2 == 2) ? dw.z
                                                                     : dw.w;
                            pk[i] &= keep_mask16(byte_lanes(wd, i % 2 == 0), p.drop.lanes_ref);
                        }
                    }
                }
            };
            auto store_P = [&](int h, const uint32_t (&pk)[32]) {
                if constexpr (F8) tmem_st16(tP + h * C::P_COLS_HALF, pk);
                else tmem_st32(tP + h * C::P_COLS_HALF, pk);
            };
#pragma unroll
            for (int k = 0; k < 4; ++k) ae[k] = ar[k] = make_float2(0.f, 0.f);
            if (kLazyMax && lazy_max) {
                // Against the running reference; P_t and O_t are free once
                // P.V_t(j-1) has completed.  Both halves are released together
                // after the overflow check.
                m_used = m_sub;
                {
                    uint32_t pk[32];
                    exp_half(0, m_sub, pk);
                    if (t == lead && lane == 0) mbar_arrive(&bars->exp_mark);
                    if (!(ok = mbar_wait_warp(&bars->pv_done[t], (j - 1) & 1, g, 23 + t))) break;
                    tc_fence_after();
                    store_P(0, pk);
                    exp_half(1, m_sub, pk);
                    store_P(1, pk);
                }
                const float2 e0 = __fadd2_rn(__fadd2_rn(ae[0], ae[1]), __fadd2_rn(ae[2], ae[3]));
                if (__any_sync(0xffffffffu, !(e0.x + e0.y <= 0x1p64f))) {
                    // Rare: this block outgrows the reference.  Move the
                    // reference to the block's max (for every row of the warp,
                    // as an ordinary rescale) and redo the block.
                    const float m_blk = row_max() * sl2;
                    if (m_blk > m_used) {
                        alpha = ex2_approx(m_used - m_blk);
                        m_used = m_blk;
                    }
                    m_sub = (m_used == -INFINITY) ? 0.f : m_used;
                    rescale_O();
                    l *= alpha;
                    lr *= alpha;
                    tmem_st_wait();  // the stores above land before their replacements
#pragma unroll
                    for (int k = 0; k < 4; ++k) ae[k] = ar[k] = make_float2(0.f, 0.f);
                    uint32_t pk[32];
                    exp_half(0, m_sub, pk);
                    store_P(0, pk);
                    exp_half(1, m_sub, pk);
                    store_P(1, pk);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&bars->p_full[t][0]);
                mbar_arrive(&bars->p_full[t][1]);
            } else {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t pk[32];
                    exp_half(h, m_sub, pk);
                    if constexpr (C::SEP) {
                        if (h == 0) {
                            if (t == lead && lane == 0) mbar_arrive(&bars->exp_mark);
                            // P_t and O_t are free once P.V_t(j-1) has completed.
                            if (j > 0) {
                                if (!(ok = mbar_wait_warp(&bars->pv_done[t], (j - 1) & 1, g, 23 + t)))
                                    break;
                                tc_fence_after();
                            }
                            rescale_O();
                        }
                    }
                    store_P(h, pk);
                    // Release this half of P: the tensor core starts on keys
                    // [64h, 64h + 64) while the other half is still being computed.
                    tmem_st_wait();
                    tc_fence_before();
                    mbar_arrive(&bars->p_full[t][h]);
                }
            }
            if (!ok) break;
            {
                const float2 e = __fadd2_rn(__fadd2_rn(ae[0], ae[1]), __fadd2_rn(ae[2], ae[3]));
                const float2 r = __fadd2_rn(__fadd2_rn(ar[0], ar[1]), __fadd2_rn(ar[2], ar[3]));
                l += e.x + e.y;
                lr += r.x + r.y;
            }
        }
        // ------------------------------------------------------------ epilogue
        if (padding_cta) {
            // Padding query rows: O = 0, LSE = 0.
            if (q < p.N) {
                __nv_bfloat16* orow = p.O + (static_cast<size_t>(bh) * p.N + q) * D;
#pragma unroll
                for (int c = 0; c < D; c += 8) st_global_v4(orow + c, 0u, 0u, 0u, 0u);
                p.LSE[static_cast<size_t>(bh) * p.N + q] = 0.f;
            }
        } else {
            // O_t is complete once its last P.V is (every warp waits; the tile's
            // four warps then meet at a named barrier whatever the outcome).
            const bool go = ok && (C::SEP ? mbar_wait_warp(&bars->pv_done[t], (nt - 1) & 1, g, 25 + t)
                                          : mbar_wait_warp(&bars->o_full[t], 0, g, 11 + t));
            if (go) tc_fence_after();
            const bool real = q < len;  // padding rows of a partly padded tile get zeros
            const float inv_l = real ? p.o_scale / lr : 0.f;
            const bool valid = q < p.N;
            if constexpr (!F8) {
                // O_t out of TMEM in one go, normalised, packed to bf16 and
                // written in the 128-byte-swizzled layout of a Q tile into Q_t's
                // own shared memory, which no MMA reads once O_t is complete
                // (its last S was issued before its last P.V, by the same
                // thread or, with P in its own columns, read by this softmax).
                // One thread then writes the tile with TMA stores, which clip
                // the rows past N.
                uint8_t* stage = smem + C::OFF_Q + t * C::TILE_BYTES;
                if (go) {
                    uint32_t o[D];
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) tmem_ld32(tO + c * 32, o + c * 32);
                    tmem_ld_wait();
                    reg_fence<D>(o);
                    const uint32_t srow = smem_u32(stage) + static_cast<uint32_t>(row) * 128u;
#pragma unroll
                    for (int u = 0; u < D / 8; ++u) {  // 16-byte units: 8 columns each
                        const uint32_t chunk = u / 8, uu = u % 8;
                        st_shared_v4(srow + chunk * 16384u + ((uu ^ (static_cast<uint32_t>(row) & 7u)) << 4),
                                     pack_bf16x2(__uint_as_float(o[8 * u + 0]) * inv_l,
                                                 __uint_as_float(o[8 * u + 1]) * inv_l),
                                     pack_bf16x2(__uint_as_float(o[8 * u + 2]) * inv_l,
                                                 __uint_as_float(o[8 * u + 3]) * inv_l),
                                     pack_bf16x2(__uint_as_float(o[8 * u + 4]) * inv_l,
                                                 __uint_as_float(o[8 * u + 5]) * inv_l),
                                     pack_bf16x2(__uint_as_float(o[8 * u + 6]) * inv_l,
                                                 __uint_as_float(o[8 * u + 7]) * inv_l));
                    }
                    fence_proxy_async_smem();
                }
                const bool tile_go = named_bar_and(1 + t, 128, go);  // the tile's four warps
                if (tile_go && warp % 4 == 0 && lane == 0) {
#pragma unroll
                    for (int c = 0; c < C::CHUNKS; ++c)
                        tma_store_3d(&mapO, stage + c * 16384, c * C::BOX_ELEMS, tile_first_q, bh);
                    bulk_commit_group();
                    bulk_wait_read_all();  // shared memory read before the CTA exits
                }
            } else if (go) {
                __nv_bfloat16* orow = p.O + (static_cast<size_t>(bh) * p.N + (valid ? q : 0)) * D;
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tO + c * 32, o);
                    tmem_ld_wait();
                    reg_fence<32>(o);
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l,
                                           __uint_as_float(o[2 * i + 1]) * inv_l);
                    if (valid) {
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            st_global_v4(orow + c * 32 + v * 8, w[4 * v], w[4 * v + 1], w[4 * v + 2],
                                         w[4 * v + 3]);
                    }
                }
            }
            if (go && valid) {
                // LSE in natural-log units: (m + log2 l) * ln 2.
                p.LSE[static_cast<size_t>(bh) * p.N + q] =
                    real ? (m_used + __log2f(l)) * 0.69314718055994531f : 0.f;
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace fa
