// fa_bwd.cuh -- exact attention backward for sm_100a (tcgen05 + TMA + TMEM).
//
// The gradient of <O, dO> for O = softmax(scale Q K^T [+causal]) V, computed
// the way unite.ai "Flash Attention: Revolutionizing Transformer Efficiency"
// (idea 2, recomputation) describes: the probabilities are not stored by the
// forward but recomputed block by block from Q, K and the saved per-row
// logsumexp.  With P_ij = exp(scale <q_i,k_j> - LSE_i):
//     dV_j = sum_i P_ij dO_i            dP_ij = <dO_i, v_j>
//     D_i  = <dO_i, O_i>                dS_ij = P_ij (dP_ij - D_i)
//     dQ_i = scale sum_j dS_ij k_j      dK_j  = scale sum_i dS_ij q_i
//
// Three launches on the caller's stream:
//   1. bwd_pre:  D_i (fp32), LSE_i * log2(e), zero the fp32 dQ accumulator
//   2. bwd_main: one CTA per (key block of 128, head); loops over query blocks
//   3. bwd_dq:   dQ = bf16(scale * dQacc)
// 2 and 3 are programmatic dependent launches: bwd_main's CTAs start (TMEM,
// barriers, K/V/Q/dO loads) while bwd_pre drains and wait (griddepcontrol)
// only before reading D, LSE2 or the accumulator; bwd_dq's CTAs wait for the
// whole of bwd_main.  What follows the three still sees them in stream order.
//
// bwd_main, per query block i (the key block j is fixed per CTA):
//   MMA1  S^T  = K_j Q_i^T            TMEM [0,128)      (lane = key)
//   MMA2  dP^T = V_j dO_i^T           TMEM [128,256)
//   MMA3  dV  += P^T dO_i             P^T bf16 in TMEM over S^T, dO MN-major
//   MMA4  dK  += dS^T Q_i             dS^T bf16 in smem (K-major), Q MN-major
//   MMA5  dQ_i = dS K_j               dS^T smem read MN-major, K MN-major
// dQ_i goes to 128-B-swizzled shared memory and is added to the fp32
// accumulator with TMA tensor reduce-adds (one per 32-column box).
// Warps: 0-7 compute (warp w: TMEM lane quarter w%4, column half w/4),
// 8 MMA issuer of S^T, dP^T and dV (TMEM owner), 9 TMA producer, 10 dQ
// reducer, 11 MMA issuer of dK and dQ.  The two issuers share the five
// products 16 : 16 instructions, so that S^T(i+1) is not held behind the
// barrier waits of dK(i) and dQ(i).
#pragma once

#include <algorithm>

#include "philox.cuh"
#include "sm100.cuh"
#include "tma_host.h"

namespace fa {

constexpr int BWD_BM = 128;  // queries per block
constexpr int BWD_BN = 128;  // keys per CTA
constexpr int BWD_THREADS = 384;  // 3 warpgroups
// Registers: launched at 168 (384 x 168 = 64512); the control warpgroup drops
// to 88 and the two compute warpgroups rise to 208: 256 x 208 + 128 x 88.
constexpr uint32_t BWD_REGS_COMPUTE = 208;
constexpr uint32_t BWD_REGS_CONTROL = 88;

inline size_t round_up_128(int n) { return (static_cast<size_t>(n) + 127) / 128 * 128; }

// Workspace: [D: BH*Npad f32][LSE2: BH*Npad f32][dQacc: BH*Npad*d f32]
//            [dQ block counters: BH*Npad/128 int32, padded to 256 B]
// The counters order the dQ additions in the deterministic mode.
inline size_t bwd_counter_bytes(int B, int H, int N) {
    const size_t n = static_cast<size_t>(B) * H * (round_up_128(N) / 128);
    return (n * 4 + 255) / 256 * 256;
}
inline size_t bwd_workspace_bytes(int B, int H, int N, int d) {
    const size_t rows = static_cast<size_t>(B) * H * round_up_128(N);
    return rows * 4 * 2 + rows * static_cast<size_t>(d) * 4 + bwd_counter_bytes(B, H, N);
}

template <int D>
struct BwdCfg {
    static constexpr int TILE = 128 * D * 2;      // bf16 tile of 128 rows
    static constexpr int QS = (D == 64) ? 2 : 1;  // Q/dO ring depth
    static constexpr int CHUNKS = D / 64;
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + TILE;
    static constexpr int OFF_Q = OFF_V + TILE;               // QS tiles
    static constexpr int OFF_DO = OFF_Q + QS * TILE;         // QS tiles
    static constexpr int OFF_DS = OFF_DO + QS * TILE;        // 128x128 bf16 = 32 KB
    static constexpr int OFF_DQ = OFF_DS + 32768;            // 128 x D fp32, D/32 swizzled boxes
    static constexpr int OFF_VEC = OFF_DQ + 128 * D * 4;     // QS x (LSE2[128], D[128])
    static constexpr int OFF_BAR = OFF_VEC + QS * 1024;
    static constexpr int BAR_BYTES = 384;
    static constexpr int SMEM_BYTES = OFF_BAR + BAR_BYTES + 1024;
    // TMEM columns
    static constexpr uint32_t T_ST = 0, T_DPT = 128, T_DV = 256, T_DK = 256 + D;
    static constexpr bool DQ_ALIAS = (D == 128);  // dQ shares the dP^T columns
    static constexpr uint32_t T_DQ = DQ_ALIAS ? T_DPT : 256 + 2 * D;
    // P^T: its own 64 columns when they exist (d = 64); over S^T otherwise,
    // which needs both column halves of a lane read before either writes.
    static constexpr bool P_ALIAS = (D == 128);
    static constexpr uint32_t T_PT = P_ALIAS ? T_ST : 256 + 3 * D;
};

struct BwdBars {
    uint64_t kv_full;
    uint64_t q_full[2], q_empty[2];
    uint64_t s_full, dp_full, p_full, ds_full, ds_empty, dq_full, dq_empty, dkdv_full;
    uint64_t pair[4];
    uint64_t dq_staged, dq_free;
};

struct BwdParams {
    const float* Dvec;   // [BH, Npad]
    const float* LSE2;   // [BH, Npad]
    float* dQacc;        // [BH, Npad, d]
    __nv_bfloat16* dK;
    __nv_bfloat16* dV;
    int N, Npad, n_q_blocks;
    int H, group;        // query heads per batch; query heads per K/V head
    int Hkv, n_kv_heads; // K/V heads per batch; B * Hkv
    const int* seqlens;  // [B] real tokens per batch (device), or null
    int* dq_count;       // [BH, Npad/128] dQ block counters (deterministic mode), or null
    float scale, scale_log2;
    int causal;
    uint32_t* err;
    DropoutParams drop;  // attention dropout (kernels instantiated with DROP only)
};

// ---------------------------------------------------------------------------
// 1. preprocess
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256)
fa_bwd_pre_kernel(const __nv_bfloat16* __restrict__ O, const __nv_bfloat16* __restrict__ dO,
                  const float* __restrict__ LSE, float* __restrict__ Dvec,
                  float* __restrict__ LSE2, float* __restrict__ dQacc, int N, int Npad,
                  long long rows_pad, const int* __restrict__ seqlens, int H,
                  int* __restrict__ dq_count, long long n_count) {
    constexpr int TPR = D / 8;  // threads per row, 8 bf16 (16 B) each
    grid_dep_launch();  // the main kernel may start its prologue
    const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    for (long long c = tid; c < n_count; c += static_cast<long long>(gridDim.x) * blockDim.x)
        dq_count[c] = 0;
    const int sub = threadIdx.x % TPR;
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x / TPR;
    for (long long r = tid / TPR; r < rows_pad; r += stride) {
        const long long bh = r / Npad;
        const int i = static_cast<int>(r % Npad);
        const int len = seqlens ? min(max(seqlens[bh / H], 0), N) : N;
        float acc = 0.f;
        if (i < len) {
            const size_t off = (static_cast<size_t>(bh) * N + i) * D + sub * 8;
            const uint4 a = *reinterpret_cast<const uint4*>(O + off);
            const uint4 b = *reinterpret_cast<const uint4*>(dO + off);
            const __nv_bfloat162* ah = reinterpret_cast<const __nv_bfloat162*>(&a);
            const __nv_bfloat162* bh2 = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 x = __bfloat1622float2(ah[k]);
                const float2 y = __bfloat1622float2(bh2[k]);
                acc = fmaf(x.x, y.x, acc);
                acc = fmaf(x.y, y.y, acc);
            }
        }
#pragma unroll
        for (int o = TPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o, TPR);
        if (sub == 0) {
            Dvec[r] = acc;
            LSE2[r] = (i < len) ? LSE[static_cast<size_t>(bh) * N + i] * 1.4426950408889634f : 0.f;
        }
        float4* z = reinterpret_cast<float4*>(dQacc + static_cast<size_t>(r) * D);
#pragma unroll
        for (int k = 0; k < D / 4 / TPR; ++k) z[sub + k * TPR] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// ---------------------------------------------------------------------------
// 3. dQ finalize
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256)
fa_bwd_dq_kernel(const float* __restrict__ dQacc, __nv_bfloat16* __restrict__ dQ, int N, int Npad,
                 float scale, long long n_vec) {
    grid_dep_wait();  // dQacc is complete only when the main kernel has finished
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < n_vec;
         e += stride) {
        const long long row = e / (D / 8);
        const int c8 = static_cast<int>(e % (D / 8)) * 8;
        const long long bh = row / N;
        const int i = static_cast<int>(row % N);
        const float4* src =
            reinterpret_cast<const float4*>(dQacc + (static_cast<size_t>(bh) * Npad + i) * D + c8);
        const float4 a = src[0], b = src[1];
        uint4 w;
        w.x = pack_bf16x2(a.x * scale, a.y * scale);
        w.y = pack_bf16x2(a.z * scale, a.w * scale);
        w.z = pack_bf16x2(b.x * scale, b.y * scale);
        w.w = pack_bf16x2(b.z * scale, b.w * scale);
        *reinterpret_cast<uint4*>(dQ + static_cast<size_t>(row) * D + c8) = w;
    }
}

// ---------------------------------------------------------------------------
// 2. main kernel
// ---------------------------------------------------------------------------
// Per query block i the compute warps do three phases:
//   P(i):   P^T = exp2(S^T * scale*log2e - LSE2[q])  (TMEM -> regs -> TMEM)
//   dS(i):  dS^T = P^T * (dP^T - D[q])               (-> swizzled smem, bf16)
//   dQr(i): dQ_i from TMEM -> swizzled fp32 smem staging for the reducer warp
// and the work is software-pipelined across the two MMA issuers:
//   compute:  P(0) dS(0) | P(1) dQr(0) dS(1) | P(2) dQr(1) dS(2) | ... dQr(n-1)
//   MMA 8:    S(0) dP(0) dV(0) S(1) dP(1) dV(1) S(2) ...   (dP(i+1) after dS(i) is read)
//   MMA 11:   dK(0) dQ(0) dK(1) dQ(1) ...                   (each after dS(i) is stored)
// so the exp work of block i+1 overlaps the dK/dQ MMAs of block i.
// DROP: attention dropout (philox.cuh).  With Pd = P z / q the forward
// output is sum_j Pd_ij v_j, so dV takes Pd^T and dS takes the dropped dP:
//     dV_j += sum_i Pd_ij dO_i,   dS_ij = P_ij (z_ij dP_ij / q - D_i)
// (D_i = <dO_i, O_i> is unchanged).  The keep bits are regenerated from the
// same counters as the forward's.
template <int D, bool DROP = false>
__global__ void __launch_bounds__(BWD_THREADS, 1)
fa_bwd_main_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                   const __grid_constant__ CUtensorMap mapV, const __grid_constant__ CUtensorMap mapdO,
                   const __grid_constant__ CUtensorMap mapdQacc, const BwdParams p) {
    using C = BwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    BwdBars* bars = reinterpret_cast<BwdBars*>(smem + C::OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + sizeof(BwdBars));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const Guard g{abort_flag, p.err};

    const uint32_t warp = warp_id(), lane = lane_id();
    // CTA = (key block, K/V head).  With grouped-query attention the CTA walks
    // every query head of its group, so dK/dV sum over the group in TMEM.
    // 1-D grid.  Causal: key-block-major, block 0 (the most query blocks) of
    // every head first, so the heaviest CTAs never form the tail.
    // Non-causal (equal work): head-major, the key blocks of one head
    // adjacent, so the CTAs resident at one time stream few heads' Q and dO.
    int kb, bkv;
    if (p.causal) {
        kb = static_cast<int>(blockIdx.x) / p.n_kv_heads;
        bkv = static_cast<int>(blockIdx.x) % p.n_kv_heads;
    } else {
        bkv = static_cast<int>(blockIdx.x) / p.n_q_blocks;
        kb = static_cast<int>(blockIdx.x) % p.n_q_blocks;
    }
    const int batch = bkv / p.Hkv;
    const int bq0 = batch * p.H + (bkv % p.Hkv) * p.group;  // first query head of the group
    const int k0 = kb * BWD_BN;
    // Padded batches: only the first len tokens are real; a key block past len
    // has zero gradients, query blocks past len contribute nothing.
    const int len = p.seqlens ? min(max(__ldg(p.seqlens + batch), 0), p.N) : p.N;
    const bool padding_cta = k0 >= len;
    const int i_begin = p.causal ? kb : 0;  // first query block that sees this key block
    const int nq = padding_cta ? 0 : (len + BWD_BM - 1) / BWD_BM - i_begin;  // per query head
    const int n_iter = nq * p.group;
    // iteration it -> (query head, query block)
    auto q_head = [&](int it) { return bq0 + it / nq; };
    auto q_block0 = [&](int it) { return (i_begin + it % nq) * BWD_BM; };

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        mbar_init(&bars->kv_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->q_full[s], 1);
            mbar_init(&bars->q_empty[s], 2);  // both MMA issuers read a Q/dO stage
        }
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->dp_full, 1);
        mbar_init(&bars->p_full, 256);
        mbar_init(&bars->ds_full, 256);
        mbar_init(&bars->ds_empty, 1);
        mbar_init(&bars->dq_full, 1);
        mbar_init(&bars->dq_empty, 256);
        mbar_init(&bars->dkdv_full, 2);  // dV from issuer 8, dK from issuer 11
        for (int q = 0; q < 4; ++q) mbar_init(&bars->pair[q], 64);
        mbar_init(&bars->dq_staged, 256);
        mbar_init(&bars->dq_free, 1);
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
    grid_dep_launch();  // the finalize kernel waits for this grid's completion

    if (warp == 9) {
        // ------------------------------------------------------------ TMA producer
        regs_decrease<BWD_REGS_CONTROL>();
        if (lane == 0 && !padding_cta) {
            tma_prefetch_desc(&mapQ);
            tma_prefetch_desc(&mapK);
            tma_prefetch_desc(&mapV);
            tma_prefetch_desc(&mapdO);
            mbar_arrive_expect_tx(&bars->kv_full, 2 * C::TILE);
#pragma unroll
            for (int c = 0; c < C::CHUNKS; ++c) {
                tma_load_3d(smem + C::OFF_K + c * 16384, &mapK, &bars->kv_full, c * 64, k0, bkv);
                tma_load_3d(smem + C::OFF_V + c * 16384, &mapV, &bars->kv_full, c * 64, k0, bkv);
            }
            int issued = 0;
            for (int it = 0; it < n_iter; ++it) {
                const int s = it % C::QS;
                const uint32_t ph = (it / C::QS) & 1;
                const int q0 = q_block0(it), bh = q_head(it);
                if (it >= C::QS && !mbar_wait(&bars->q_empty[s], ph ^ 1, g, 21)) break;
                mbar_arrive_expect_tx(&bars->q_full[s], 2 * C::TILE + 1024);
#pragma unroll
                for (int c = 0; c < C::CHUNKS; ++c) {
                    tma_load_3d(smem + C::OFF_Q + s * C::TILE + c * 16384, &mapQ, &bars->q_full[s],
                                c * 64, q0, bh);
                    tma_load_3d(smem + C::OFF_DO + s * C::TILE + c * 16384, &mapdO,
                                &bars->q_full[s], c * 64, q0, bh);
                }
                // D and LSE2 come from the preprocess kernel (launched before
                // this one, which may have started before it finished).
                if (it == 0) grid_dep_wait();
                const size_t voff = static_cast<size_t>(bh) * p.Npad + q0;
                bulk_load(smem + C::OFF_VEC + s * 1024, p.LSE2 + voff, 512, &bars->q_full[s]);
                bulk_load(smem + C::OFF_VEC + s * 1024 + 512, p.Dvec + voff, 512, &bars->q_full[s]);
                issued = it + 1;
            }
            mbar_drain(&bars->kv_full, 0);
            for (int it = max(0, issued - C::QS); it < issued; ++it)
                mbar_drain(&bars->q_full[it % C::QS], (it / C::QS) & 1);
        }
    } else if (warp == 8 || warp == 11) {
        // ------------------------------------------------------------ MMA issuers
        regs_decrease<BWD_REGS_CONTROL>();
        if (!padding_cta) {  // the whole warp; one elected lane issues
            const uint32_t id_s = idesc_bf16(128, 128, false, false);  // S^T, dP^T
            const uint32_t id_kn = idesc_bf16(128, D, false, true);    // dV, dK (B MN-major)
            const uint32_t id_q = idesc_bf16(128, D, true, true);      // dQ (A, B MN-major)
            const uint32_t sK = smem_u32(smem + C::OFF_K), sV = smem_u32(smem + C::OFF_V);
            const uint32_t sDS = smem_u32(smem + C::OFF_DS);
            auto sQ = [&](int it) { return smem_u32(smem + C::OFF_Q + (it % C::QS) * C::TILE); };
            auto sdO = [&](int it) { return smem_u32(smem + C::OFF_DO + (it % C::QS) * C::TILE); };
            auto q_wait = [&](int it, uint32_t site) {
                return mbar_wait_warp(&bars->q_full[it % C::QS], (it / C::QS) & 1, g, site);
            };
            if (warp == 8) {
                // S^T(it), dP^T(it), dV(it).  Program order covers the TMEM
                // reuse of S^T / P^T: S^T(it+1) follows dV(it), which followed
                // P^T(it) being written, i.e. S^T(it) being read.
                auto mma_S = [&](int it) {  // S^T = K Q^T
                    mma_ss_blk<D / 16, FA_STEP_KMAJOR, FA_STEP_KMAJOR>(
                        tmem + C::T_ST, sdesc_sw128(sK, 16, 1024), sdesc_sw128(sQ(it), 16, 1024), id_s, 0u);
                    tc_commit_w(&bars->s_full);
                };
                auto mma_dP = [&](int it) {  // dP^T = V dO^T
                    mma_ss_blk<D / 16, FA_STEP_KMAJOR, FA_STEP_KMAJOR>(
                        tmem + C::T_DPT, sdesc_sw128(sV, 16, 1024), sdesc_sw128(sdO(it), 16, 1024), id_s, 0u);
                    tc_commit_w(&bars->dp_full);
                };
                auto mma_dV = [&](int it) {  // dV += P^T dO   (P^T from TMEM)
                    mma_ts_blk<8, 8, 128>(tmem + C::T_DV, tmem + C::T_PT,
                                          sdesc_sw128(sdO(it), 16384, 1024), id_kn, it > 0 ? 1u : 0u);
                    tc_commit_w(&bars->q_empty[it % C::QS]);  // this issuer is done with the stage
                };
                bool ok = mbar_wait_warp(&bars->kv_full, 0, g, 22) && q_wait(0, 23);
                if (ok) {
                    tc_fence_after();
                    mma_S(0);
                    mma_dP(0);
                }
                for (int it = 0; ok && it < n_iter; ++it) {
                    const bool more = it + 1 < n_iter;
                    if (!(ok = mbar_wait_warp(&bars->p_full, it & 1, g, 25))) break;
                    tc_fence_after();
                    mma_dV(it);
                    if (!more) break;
                    if (!(ok = q_wait(it + 1, 23))) break;
                    tc_fence_after();
                    mma_S(it + 1);
                    // dP^T(it+1) overwrites dP^T(it): the compute warps must
                    // have read it (ds_full), and where dQ shares those columns
                    // (d = 128) they must also have read dQ(it).
                    if (!(ok = mbar_wait_warp(&bars->ds_full, it & 1, g, 26))) break;
                    if (C::DQ_ALIAS && !(ok = mbar_wait_warp(&bars->dq_empty, it & 1, g, 24))) break;
                    tc_fence_after();
                    mma_dP(it + 1);
                }
                if (ok) tc_commit_w(&bars->dkdv_full);
            } else {
                // dK(it), dQ(it) from dS(it) in shared memory.
                bool ok = mbar_wait_warp(&bars->kv_full, 0, g, 37);
                for (int it = 0; ok && it < n_iter; ++it) {
                    if (!(ok = q_wait(it, 38))) break;
                    if (!(ok = mbar_wait_warp(&bars->ds_full, it & 1, g, 39))) break;
                    // dQ(it) overwrites dQ(it-1) in its own columns (d = 64)...
                    if (!C::DQ_ALIAS && it > 0 && !(ok = mbar_wait_warp(&bars->dq_empty, (it - 1) & 1, g, 27)))
                        break;
                    // ...or dP^T(it), which ds_full shows read (d = 128).
                    tc_fence_after();
                    // dK += dS^T Q
                    mma_ss_blk<8, FA_STEP_KMAJOR, 128>(tmem + C::T_DK, sdesc_sw128(sDS, 16, 1024),
                                                       sdesc_sw128(sQ(it), 16384, 1024), id_kn,
                                                       it > 0 ? 1u : 0u);
                    // dQ = dS K
                    mma_ss_blk<8, 128, 128>(tmem + C::T_DQ, sdesc_sw128(sDS, 16384, 1024),
                                            sdesc_sw128(sK, 16384, 1024), id_q, 0u);
                    tc_commit_w(&bars->dq_full);
                    tc_commit_w(&bars->ds_empty);
                    tc_commit_w(&bars->q_empty[it % C::QS]);
                }
                if (ok) tc_commit_w(&bars->dkdv_full);
            }
        }
    } else if (warp == 10) {
        // ------------------------------------------------------------ dQ reducer
        regs_decrease<BWD_REGS_CONTROL>();
        if (lane == 0) {
            tma_prefetch_desc(&mapdQacc);
            grid_dep_wait();  // dQacc and the counters are zeroed by the preprocess kernel
            // Deterministic mode: the additions into one dQ block are made in
            // ascending key-block order.  Before adding, wait until the block's
            // counter equals this CTA's key block (every earlier key block of
            // the same head has added and published); after the addition has
            // fully completed, publish by incrementing the counter.  Only CTAs
            // with a lower grid index are waited for (both CTA orders put a
            // head's lower key blocks first), so the waits always end.
            const bool det = p.dq_count != nullptr;
            for (int it = 0; it < n_iter; ++it) {
                if (!mbar_wait(&bars->dq_staged, it & 1, g, 28)) break;
                const int q0 = q_block0(it), bh = q_head(it);
                int* cnt = det ? p.dq_count + static_cast<size_t>(bh) * p.n_q_blocks + q0 / BWD_BM
                               : nullptr;
                if (det) {
                    if (!wait_counter(cnt, kb, g, 31)) break;
                    fence_proxy_async_global();
                }
#pragma unroll
                for (int b = 0; b < D / 32; ++b)
                    tma_reduce_add_3d(&mapdQacc, smem + C::OFF_DQ + b * 16384, b * 32, q0, bh);
                bulk_commit_group();
                bulk_wait_read_all();
                mbar_arrive(&bars->dq_free);
                if (det) {
                    bulk_wait_all();
                    __threadfence();
                    fence_proxy_async_global();
                    counter_release_add(cnt);
                }
            }
            bulk_wait_all();
        }
    } else {
        // ------------------------------------------------------------ compute warps 0-7
        regs_increase<BWD_REGS_COMPUTE>();
        const uint32_t quarter = warp % 4, half = warp / 4;
        const uint32_t lane_base = quarter * 32;
        const int r = lane_base + lane;  // TMEM lane: key row (P, dS) or query row (dQ)
        const int key = k0 + r;
        const float sl2 = p.scale_log2;
        const uint32_t sDSrow = smem_u32(smem + C::OFF_DS + half * 16384) + r * 128;
        const uint32_t sDQ = smem_u32(smem + C::OFF_DQ);
        float pv[64];  // P^T (then dS^T) for this thread's 64 queries
        uint32_t keep_lo = ~0u, keep_hi = ~0u;  // dropout keep bits of those queries
        auto kept = [&](int c) { return (((c < 32) ? keep_lo : keep_hi) >> keep_bit_index(c & 31)) & 1u; };
        bool ok = true;

        // ---- P(it): P^T = exp2(S^T * scale*log2e - LSE2[q])
        auto phase_P = [&](int it) -> bool {
            const int s = it % C::QS;
            const uint32_t ph = (it / C::QS) & 1;
            const int q0 = q_block0(it);
            const int qh = q0 + 64 * half;  // first query of this warp's columns
            if constexpr (DROP) {
                // Made before S^T is ready: they depend only on the indices.
                const uint2 M = keep_bits_key_row(p.drop, static_cast<uint32_t>(key),
                                                  static_cast<uint32_t>(qh),
                                                  static_cast<uint32_t>(q_head(it)), lane);
                keep_lo = M.x;
                keep_hi = M.y;
            }
            if (!mbar_wait(&bars->q_full[s], ph, g, 29)) return false;
            if (!mbar_wait_warp(&bars->s_full, it & 1, g, 30)) return false;
            tc_fence_after();
            {
                uint32_t u[64];
                tmem_ld32(tmem_addr(tmem, lane_base, C::T_ST + 64 * half), u);
                tmem_ld32(tmem_addr(tmem, lane_base, C::T_ST + 64 * half + 32), u + 32);
                tmem_ld_wait();
                reg_fence<64>(u);
#pragma unroll
                for (int c = 0; c < 64; ++c) pv[c] = __uint_as_float(u[c]);
            }
            const uint32_t vL = smem_u32(smem + C::OFF_VEC + s * 1024) + 256 * half;
            const bool need_mask =
                (key >= len) || (q0 + BWD_BM > len) || (p.causal && qh < k0 + BWD_BN);
#pragma unroll
            for (int c4 = 0; c4 < 16; ++c4) {
                const float4 l4 = ld_shared_v4f(vL + 16 * c4);
                const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int c = 4 * c4 + e;
                    pv[c] = ex2_approx(fmaf(pv[c], sl2, -lv[e]));
                }
            }
            if (need_mask) {
                const int qlim = p.causal ? key : 0;   // causal: keep q >= key
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    const int q = qh + c;
                    if (key >= len || q >= len || q < qlim) pv[c] = 0.f;
                }
            }
            if (C::P_ALIAS) {
                // Both column halves of these lanes must have read S^T before
                // P^T (which overlaps it) is written.
                mbar_arrive(&bars->pair[quarter]);
                if (!mbar_wait_warp(&bars->pair[quarter], it & 1, g, 31)) return false;
            }
            {
                uint32_t pk[32];
                if constexpr (DROP) {
                    const float ks = p.drop.keep_scale;
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        pk[c] = pack_bf16x2(kept(2 * c) ? pv[2 * c] * ks : 0.f,
                                            kept(2 * c + 1) ? pv[2 * c + 1] * ks : 0.f);
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c) pk[c] = pack_bf16x2(pv[2 * c], pv[2 * c + 1]);
                }
                tmem_st32(tmem_addr(tmem, lane_base, C::T_PT + 32 * half), pk);
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&bars->p_full);
            return true;
        };
        // ---- dS(it): dS^T = P^T * (dP^T - D[q]) -> swizzled bf16 smem
        auto phase_dS = [&](int it) -> bool {
            const int s = it % C::QS;
            if (!mbar_wait_warp(&bars->dp_full, it & 1, g, 32)) return false;
            tc_fence_after();
            const uint32_t vD = smem_u32(smem + C::OFF_VEC + s * 1024) + 512 + 256 * half;
            {
                uint32_t u[64];
                tmem_ld32(tmem_addr(tmem, lane_base, C::T_DPT + 64 * half), u);
                tmem_ld32(tmem_addr(tmem, lane_base, C::T_DPT + 64 * half + 32), u + 32);
                tmem_ld_wait();
                reg_fence<64>(u);
#pragma unroll
                for (int c4 = 0; c4 < 16; ++c4) {
                    const float4 d4 = ld_shared_v4f(vD + 16 * c4);
                    const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int c = 4 * c4 + e;
                        float dp = __uint_as_float(u[c]);
                        if constexpr (DROP) dp = kept(c) ? dp * p.drop.keep_scale : 0.f;
                        pv[c] = pv[c] * (dp - dv[e]);
                    }
                }
            }
            tc_fence_before();
            if (it > 0 && !mbar_wait(&bars->ds_empty, (it - 1) & 1, g, 33)) return false;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                st_shared_v4(sDSrow + ((cc ^ (r & 7)) << 4), pack_bf16x2(pv[8 * cc + 0], pv[8 * cc + 1]),
                             pack_bf16x2(pv[8 * cc + 2], pv[8 * cc + 3]),
                             pack_bf16x2(pv[8 * cc + 4], pv[8 * cc + 5]),
                             pack_bf16x2(pv[8 * cc + 6], pv[8 * cc + 7]));
            }
            fence_proxy_async_smem();
            mbar_arrive(&bars->ds_full);
            return true;
        };
        // ---- dQr(it): dQ_i (lane = query) -> 128-B-swizzled fp32 staging, one
        // 32-column box (16 KB) per 128 B of each row; the reducer adds it to
        // the fp32 accumulator with TMA reduce-add.
        auto phase_dQr = [&](int it) -> bool {
            constexpr int HC = D / 2;  // columns of dQ this warp reads
            if (!mbar_wait_warp(&bars->dq_full, it & 1, g, 34)) return false;
            tc_fence_after();
            uint32_t u[HC];
#pragma unroll
            for (int c = 0; c < HC; c += 32)
                tmem_ld32(tmem_addr(tmem, lane_base, C::T_DQ + HC * half + c), u + c);
            tmem_ld_wait();
            reg_fence<HC>(u);
            tc_fence_before();
            mbar_arrive(&bars->dq_empty);
            if (it > 0 && !mbar_wait(&bars->dq_free, (it - 1) & 1, g, 35)) return false;
#pragma unroll
            for (int b = 0; b < HC / 32; ++b) {
                const uint32_t row = sDQ + (HC / 32 * half + b) * 16384 + r * 128;
#pragma unroll
                for (int cc = 0; cc < 8; ++cc)
                    st_shared_v4(row + ((cc ^ (r & 7)) << 4), u[32 * b + 4 * cc],
                                 u[32 * b + 4 * cc + 1], u[32 * b + 4 * cc + 2],
                                 u[32 * b + 4 * cc + 3]);
            }
            fence_proxy_async_smem();
            mbar_arrive(&bars->dq_staged);
            return true;
        };

        if (n_iter > 0) ok = phase_P(0) && phase_dS(0);
        for (int it = 1; ok && it < n_iter; ++it)
            ok = phase_P(it) && phase_dQr(it - 1) && phase_dS(it);
        if (ok && n_iter > 0) ok = phase_dQr(n_iter - 1);

        // ---- dK, dV epilogue (lane = key)
        if (padding_cta) {
            constexpr int HC = D / 2;
            if (key < p.N) {
                const size_t off = (static_cast<size_t>(bkv) * p.N + key) * D + HC * half;
#pragma unroll
                for (int c = 0; c < HC; c += 8) {
                    st_global_v4(p.dV + off + c, 0u, 0u, 0u, 0u);
                    st_global_v4(p.dK + off + c, 0u, 0u, 0u, 0u);
                }
            }
        } else if (ok && mbar_wait_warp(&bars->dkdv_full, 0, g, 36)) {
            tc_fence_after();
            constexpr int HC = D / 2;
            const bool valid = key < p.N;
            const size_t off = (static_cast<size_t>(bkv) * p.N + (valid ? key : 0)) * D + HC * half;
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                const uint32_t col = (which == 0 ? C::T_DV : C::T_DK) + HC * half;
                const float mul = which == 0 ? 1.f : p.scale;
                __nv_bfloat16* dst = (which == 0 ? p.dV : p.dK) + off;
#pragma unroll
                for (int c = 0; c < HC; c += 32) {
                    uint32_t u[32];
                    tmem_ld32(tmem_addr(tmem, lane_base, col + c), u);
                    tmem_ld_wait();
                    reg_fence<32>(u);
                    uint32_t w[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        w[k] = pack_bf16x2(__uint_as_float(u[2 * k]) * mul,
                                           __uint_as_float(u[2 * k + 1]) * mul);
                    if (valid) {
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            st_global_v4(dst + c + 8 * v, w[4 * v], w[4 * v + 1], w[4 * v + 2],
                                         w[4 * v + 3]);
                    }
                }
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

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
template <int D, bool DROP>
inline bool bwd_set_attributes_t() {
    return cudaFuncSetAttribute(fa_bwd_main_kernel<D, DROP>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                BwdCfg<D>::SMEM_BYTES) == cudaSuccess;
}

inline bool bwd_set_attributes(int d, bool drop) {
    if (d == 64) return drop ? bwd_set_attributes_t<64, true>() : bwd_set_attributes_t<64, false>();
    return drop ? bwd_set_attributes_t<128, true>() : bwd_set_attributes_t<128, false>();
}

template <int D, bool DROP>
bool bwd_launch_t(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                  const float* LSE, void* dQ, void* dK, void* dV, void* workspace, int B, int H,
                  int Hkv, int N, const int* seqlens, float scale, int causal, uint32_t* err,
                  const DropoutParams& drop, bool deterministic, cudaStream_t stream) {
    const int Npad = static_cast<int>(round_up_128(N));
    const long long rows_pad = static_cast<long long>(B) * H * Npad;
    float* Dvec = static_cast<float*>(workspace);
    float* LSE2 = Dvec + rows_pad;
    float* dQacc = LSE2 + rows_pad;
    int* dq_count = reinterpret_cast<int*>(dQacc + rows_pad * D);
    const long long n_count = deterministic ? rows_pad / 128 : 0;
    {
        const long long threads = rows_pad * (D / 8);
        const int blocks = static_cast<int>(std::min<long long>((threads + 255) / 256, 148LL * 16));
        fa_bwd_pre_kernel<D><<<blocks, 256, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(O), static_cast<const __nv_bfloat16*>(dO), LSE, Dvec,
            LSE2, dQacc, N, Npad, rows_pad, seqlens, H, dq_count, n_count);
        if (cudaGetLastError() != cudaSuccess) return false;
    }
    {
        CUtensorMap mq, mk, mv, mdo, mdq;
        const uint64_t depth = static_cast<uint64_t>(B) * H;
        const uint64_t depth_kv = static_cast<uint64_t>(B) * Hkv;
        if (!make_map_bf16_3d(&mq, Q, depth, N, D, 128) || !make_map_bf16_3d(&mk, K, depth_kv, N, D, 128) ||
            !make_map_bf16_3d(&mv, V, depth_kv, N, D, 128) || !make_map_bf16_3d(&mdo, dO, depth, N, D, 128) ||
            !make_map_f32_3d_sw128(&mdq, dQacc, depth, Npad, D))
            return false;
        BwdParams p;
        p.Dvec = Dvec;
        p.LSE2 = LSE2;
        p.dQacc = dQacc;
        p.dK = static_cast<__nv_bfloat16*>(dK);
        p.dV = static_cast<__nv_bfloat16*>(dV);
        p.N = N;
        p.Npad = Npad;
        p.n_q_blocks = Npad / 128;
        p.H = H;
        p.group = H / Hkv;
        p.Hkv = Hkv;
        p.n_kv_heads = B * Hkv;
        p.seqlens = seqlens;
        p.dq_count = deterministic ? dq_count : nullptr;
        p.scale = scale;
        p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
        p.causal = causal ? 1 : 0;
        p.err = err;
        p.drop = drop;
        const long long n_ctas = static_cast<long long>(Npad / 128) * B * Hkv;
        if (n_ctas > 0x7fffffffLL) return false;
        cudaLaunchAttribute pdl[1];
        pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        pdl[0].val.programmaticStreamSerializationAllowed = 1;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(n_ctas));
        cfg.blockDim = dim3(BWD_THREADS);
        cfg.dynamicSmemBytes = BwdCfg<D>::SMEM_BYTES;
        cfg.stream = stream;
        cfg.attrs = pdl;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, fa_bwd_main_kernel<D, DROP>, mq, mk, mv, mdo, mdq, p) !=
            cudaSuccess)
            return false;
    }
    {
        const long long n_vec = static_cast<long long>(B) * H * N * (D / 8);
        const int blocks = static_cast<int>(std::min<long long>((n_vec + 255) / 256, 148LL * 16));
        cudaLaunchAttribute pdl[1];
        pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        pdl[0].val.programmaticStreamSerializationAllowed = 1;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(blocks);
        cfg.blockDim = dim3(256);
        cfg.stream = stream;
        cfg.attrs = pdl;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, fa_bwd_dq_kernel<D>, static_cast<const float*>(dQacc),
                               static_cast<__nv_bfloat16*>(dQ), N, Npad, scale, n_vec) != cudaSuccess)
            return false;
    }
    return true;
}

// drop = null: no dropout.
inline bool bwd_launch(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                       const float* LSE, void* dQ, void* dK, void* dV, void* workspace, int B, int H,
                       int Hkv, int N, int d, const int* seqlens, float scale, int causal,
                       uint32_t* err, const DropoutParams* drop, cudaStream_t stream,
                       bool deterministic = false) {
    const DropoutParams none{};
    const DropoutParams& dp = drop ? *drop : none;
#define FA_BWD_LAUNCH(DD, DR)                                                                    \
    bwd_launch_t<DD, DR>(Q, K, V, O, dO, LSE, dQ, dK, dV, workspace, B, H, Hkv, N, seqlens, scale, \
                         causal, err, dp, deterministic, stream)
    if (d == 128) return drop ? FA_BWD_LAUNCH(128, true) : FA_BWD_LAUNCH(128, false);
    return drop ? FA_BWD_LAUNCH(64, true) : FA_BWD_LAUNCH(64, false);
#undef FA_BWD_LAUNCH
}

}  // namespace fa
