// fa_api.cu -- the C ABI (include/fa.h): argument validation, TMA descriptor
// creation and kernel launch.  All arithmetic of the attention path runs in
// the kernels of fa_fwd.cuh / fa_bwd.cuh.
#include <cmath>
#include <cstdint>
#include <mutex>

#include "fa.h"
#include "fa_bwd.cuh"
#include "fa_fwd.cuh"
#include "tma_host.h"

namespace fa {

// Per-device error word written by bounded waits that gave up (0 = none).
__device__ uint32_t g_err_word;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
    bool checked = false;
    bool supported = false;
    uint32_t* err = nullptr;  // device address of g_err_word on this device
    // d = 64, d = 128, d = 128 E4M3, d = 64 dropout, d = 128 dropout
    bool fwd_attr[5] = {false, false, false, false, false};
    bool bwd_attr[4] = {false, false, false, false};  // d = 64, 128; then with dropout
};

DeviceState g_dev[kMaxDevices];
std::mutex g_mu;

// Returns the state of the current device, or null if it is not a usable sm_100 part.
DeviceState* current_device(fa_status* st) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        *st = FA_ERR_CUDA;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState& s = g_dev[dev];
    if (!s.checked) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
            *st = FA_ERR_CUDA;
            return nullptr;
        }
        s.supported = (major == 10 && minor == 0);
        if (s.supported) {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_err_word) != cudaSuccess) {
                *st = FA_ERR_CUDA;
                return nullptr;
            }
            s.err = static_cast<uint32_t*>(p);
        }
        s.checked = true;
    }
    if (!s.supported) {
        *st = FA_ERR_UNSUPPORTED;
        return nullptr;
    }
    *st = FA_OK;
    return &s;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fa_status check_shape(int B, int H, int N, int d, float scale) {
    if (B < 1 || H < 1 || N < 1 || d < 1) return FA_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    const int64_t total = static_cast<int64_t>(B) * H * N * d;
    if (total >= (int64_t(1) << 31) || static_cast<int64_t>(B) * H > 65535LL * 65535LL)
        return FA_ERR_UNSUPPORTED;
    if (H > 65535 || B > 65535) return FA_ERR_UNSUPPORTED;
    return FA_OK;
}

// H_kv: K/V heads per batch (H_kv divides H; H_kv == H is plain multi-head).
fa_status check_heads(int H, int Hkv) {
    if (Hkv < 1 || Hkv > H || H % Hkv != 0) return FA_ERR_INVALID_ARG;
    return FA_OK;
}

// Attention-dropout parameters from (p, seed, offset): keep threshold
// t = floor((1 - p) 2^8 + 1/2) on 8-bit uniforms, keep scale 2^8 / t, and the
// Philox round keys.  *on = false when t = 2^8 (p < 2^-9: nothing is ever
// dropped), which runs the kernels without dropout; t = 0 is rejected.
fa_status make_dropout(float p, uint64_t seed, uint32_t offset, DropoutParams* d, bool* on) {
    if (!(p >= 0.f && p < 1.f)) return FA_ERR_INVALID_ARG;  // also rejects NaN
    const double t = std::floor((1.0 - static_cast<double>(p)) * 256.0 + 0.5);
    if (t < 1.0) return FA_ERR_INVALID_ARG;
    *on = t < 256.0;
    uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
    for (int r = 0; r < PHILOX_ROUNDS; ++r) {
        d->key[2 * r] = k0;
        d->key[2 * r + 1] = k1;
        k0 += 0x9E3779B9u;  // Weyl increments of Philox-4x32
        k1 += 0xBB67AE85u;
    }
    d->offset = offset;
    const uint32_t ref = 0x8000u + static_cast<uint32_t>(t) - 1u;
    d->lanes_ref = ref | (ref << 16);
    d->keep_scale = static_cast<float>(256.0 / t);
    return FA_OK;
}

// scale_qk multiplies the scores (dequant scales of E4M3 Q and K), scale_v
// the output (dequant scale of E4M3 V); both 1 for bf16 inputs.  DROP: drop
// holds the dropout parameters.
template <int D, bool F8, bool DROP = false>
fa_status launch_forward(DeviceState* ds, const void* Q, const void* K, const void* V, void* O,
                         float* LSE, int B, int H, int Hkv, int N, const int* seqlens,
                         float scale, int causal, cudaStream_t stream, double scale_qk = 1.0,
                         float scale_v = 1.f, const DropoutParams* drop = nullptr) {
    using C = FwdCfg<D, F8>;
    CUtensorMap mq, mk, mv, mo;
    const uint64_t depth = static_cast<uint64_t>(B) * H;
    const uint64_t depth_kv = static_cast<uint64_t>(B) * Hkv;
    const bool maps_ok =
        F8 ? (make_map_u8_3d(&mq, Q, depth, N, D, FWD_BM) &&
              make_map_u8_3d(&mk, K, depth_kv, N, D, FWD_BN) &&
              make_map_u8_3d(&mv, V, depth_kv, N, D, FWD_BN))
           : (make_map_bf16_3d(&mq, Q, depth, N, D, FWD_BM) &&
              make_map_bf16_3d(&mk, K, depth_kv, N, D, FWD_BN) &&
              make_map_bf16_3d(&mv, V, depth_kv, N, D, FWD_BN));
    // O (bf16 in every variant) is written by TMA stores of Q-shaped tiles.
    if (!maps_ok || !make_map_bf16_3d(&mo, O, depth, N, D, FWD_BM)) return FA_ERR_CUDA;
    const int di = F8 ? 2 : ((D == 128) ? 1 : 0) + (DROP ? 3 : 0);
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!ds->fwd_attr[di]) {
            if (cudaFuncSetAttribute(fa_fwd_kernel<D, F8, DROP>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     C::SMEM_BYTES) != cudaSuccess)
                return FA_ERR_CUDA;
            ds->fwd_attr[di] = true;
        }
    }
    FwdParams p;
    p.O = static_cast<__nv_bfloat16*>(O);
    p.LSE = LSE;
    p.N = N;
    p.n_kv_blocks = (N + FWD_BN - 1) / FWD_BN;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * scale_qk * 1.4426950408889634);
    p.o_scale = scale_v;
    p.drop = DropoutParams{};
    if (DROP) {
        p.drop = *drop;
        p.o_scale = scale_v * drop->keep_scale;
    }
    p.causal = causal ? 1 : 0;
    p.err = ds->err;
    p.n_heads = B * H;
    p.H = H;
    p.group = H / Hkv;
    p.seqlens = seqlens;
    p.n_pairs = (N + 2 * FWD_BM - 1) / (2 * FWD_BM);
    const long long n_ctas = static_cast<long long>(p.n_pairs) * p.n_heads;
    if (n_ctas > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
    dim3 grid(static_cast<unsigned>(n_ctas));
    fa_fwd_kernel<D, F8, DROP><<<grid, FWD_THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, mo, p);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

bool ensure_bwd_attributes(DeviceState* ds, int d, bool drop) {
    std::lock_guard<std::mutex> lock(g_mu);
    const int di = ((d == 128) ? 1 : 0) + (drop ? 2 : 0);
    if (!ds->bwd_attr[di]) {
        if (!bwd_set_attributes(d, drop)) return false;
        ds->bwd_attr[di] = true;
    }
    return true;
}

// Self-test of the bounded-wait path: warp 0 waits, with a short limit, on a
// barrier that nothing ever arrives at, so it gives up and records
// DEV_TIMEOUT_BASE + SELFTEST_SITE; warp 1 waits on the same barrier with the
// kernels' normal limit and must be released early by the abort flag.
constexpr uint32_t SELFTEST_SITE = 0x63;

__global__ void __launch_bounds__(64)
fa_selftest_wait_kernel(uint32_t* err, unsigned long long timeout_ns, int* released) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    const Guard g{&abort_flag, err};
    bool ok;
    if (warp_id() == 0)
        ok = mbar_wait(&bar, 0, g, SELFTEST_SITE, timeout_ns);
    else
        ok = mbar_wait(&bar, 0, g, SELFTEST_SITE + 1);
    if (!ok && warp_id() == 1 && lane_id() == 0 && released) *released = 1;
}

}  // namespace
}  // namespace fa

using namespace fa;

extern "C" {

fa_status fa_forward_dropout(const void* Q, const void* K, const void* V, void* O, float* LSE,
                             const int* seqlens, int B, int H, int H_kv, int N, int d,
                             float scale, int causal, float dropout_p, unsigned long long seed,
                             unsigned int offset, cudaStream_t stream) {
    DropoutParams drop;
    bool on = false;
    fa_status st = make_dropout(dropout_p, seed, offset, &drop, &on);
    if (st != FA_OK) return st;
    if (!on) return fa_forward_varlen(Q, K, V, O, LSE, seqlens, B, H, H_kv, N, d, scale, causal,
                                      stream);
    if (!Q || !K || !V || !O || !LSE) return FA_ERR_INVALID_ARG;
    if (seqlens && (reinterpret_cast<uintptr_t>(seqlens) & 3u)) return FA_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE))
        return FA_ERR_INVALID_ARG;
    if ((st = check_shape(B, H, N, d, scale)) != FA_OK) return st;
    if ((st = check_heads(H, H_kv)) != FA_OK) return st;
    DeviceState* ds = current_device(&st);
    if (!ds) return st;
    return d == 128 ? launch_forward<128, false, true>(ds, Q, K, V, O, LSE, B, H, H_kv, N, seqlens,
                                                       scale, causal, stream, 1.0, 1.f, &drop)
                    : launch_forward<64, false, true>(ds, Q, K, V, O, LSE, B, H, H_kv, N, seqlens,
                                                      scale, causal, stream, 1.0, 1.f, &drop);
}

fa_status fa_forward_varlen(const void* Q, const void* K, const void* V, void* O, float* LSE,
                            const int* seqlens, int B, int H, int H_kv, int N, int d,
                            float scale, int causal, cudaStream_t stream) {
    if (!Q || !K || !V || !O || !LSE) return FA_ERR_INVALID_ARG;
    if (seqlens && (reinterpret_cast<uintptr_t>(seqlens) & 3u)) return FA_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE))
        return FA_ERR_INVALID_ARG;
    fa_status st = check_shape(B, H, N, d, scale);
    if (st != FA_OK) return st;
    if ((st = check_heads(H, H_kv)) != FA_OK) return st;
    DeviceState* ds = current_device(&st);
    if (!ds) return st;
    return d == 128 ? launch_forward<128, false>(ds, Q, K, V, O, LSE, B, H, H_kv, N, seqlens,
                                                 scale, causal, stream)
                    : launch_forward<64, false>(ds, Q, K, V, O, LSE, B, H, H_kv, N, seqlens,
                                                scale, causal, stream);
}

fa_status fa_forward_fp8(const void* Q8, const void* K8, const void* V8, void* O, float* LSE,
                         float descale_q, float descale_k, float descale_v, int B, int H,
                         int H_kv, int N, int d, float scale, int causal, cudaStream_t stream) {
    if (!Q8 || !K8 || !V8 || !O || !LSE) return FA_ERR_INVALID_ARG;
    if (!aligned16(Q8) || !aligned16(K8) || !aligned16(V8) || !aligned16(O) || !aligned16(LSE))
        return FA_ERR_INVALID_ARG;
    fa_status st = check_shape(B, H, N, d, scale);
    if (st != FA_OK) return st;
    if ((st = check_heads(H, H_kv)) != FA_OK) return st;
    for (float f : {descale_q, descale_k, descale_v})
        if (!std::isfinite(f) || !(f > 0.f)) return FA_ERR_INVALID_ARG;
    if (d != 128) return FA_ERR_UNSUPPORTED;
    DeviceState* ds = current_device(&st);
    if (!ds) return st;
    return launch_forward<128, true>(ds, Q8, K8, V8, O, LSE, B, H, H_kv, N, nullptr, scale,
                                     causal, stream,
                                     static_cast<double>(descale_q) * descale_k, descale_v);
}

fa_status fa_forward_gqa(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                         int H, int H_kv, int N, int d, float scale, int causal,
                         cudaStream_t stream) {
    return fa_forward_varlen(Q, K, V, O, LSE, nullptr, B, H, H_kv, N, d, scale, causal, stream);
}

fa_status fa_forward(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                     int H, int N, int d, float scale, int causal, cudaStream_t stream) {
    return fa_forward_gqa(Q, K, V, O, LSE, B, H, H, N, d, scale, causal, stream);
}

size_t fa_backward_workspace_bytes(int B, int H, int N, int d) {
    if (check_shape(B, H, N, d, 1.f) != FA_OK) return 0;
    return bwd_workspace_bytes(B, H, N, d);
}

fa_status fa_backward_dropout(const void* Q, const void* K, const void* V, const void* O,
                              const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                              void* workspace, size_t workspace_bytes, const int* seqlens, int B,
                              int H, int H_kv, int N, int d, float scale, int causal,
                              float dropout_p, unsigned long long seed, unsigned int offset,
                              cudaStream_t stream) {
    DropoutParams drop;
    bool on = false;
    fa_status st = make_dropout(dropout_p, seed, offset, &drop, &on);
    if (st != FA_OK) return st;
    if (!Q || !K || !V || !O || !dO || !LSE || !dQ || !dK || !dV || !workspace)
        return FA_ERR_INVALID_ARG;
    if (seqlens && (reinterpret_cast<uintptr_t>(seqlens) & 3u)) return FA_ERR_INVALID_ARG;
    const void* ptrs[] = {Q, K, V, O, dO, LSE, dQ, dK, dV, workspace};
    for (const void* p : ptrs)
        if (!aligned16(p)) return FA_ERR_INVALID_ARG;
    if ((st = check_shape(B, H, N, d, scale)) != FA_OK) return st;
    if ((st = check_heads(H, H_kv)) != FA_OK) return st;
    if (workspace_bytes < bwd_workspace_bytes(B, H, N, d)) return FA_ERR_INVALID_ARG;
    DeviceState* ds = current_device(&st);
    if (!ds) return st;
    if (!ensure_bwd_attributes(ds, d, on)) return FA_ERR_CUDA;
    return bwd_launch(Q, K, V, O, dO, LSE, dQ, dK, dV, workspace, B, H, H_kv, N, d, seqlens,
                      scale, causal, ds->err, on ? &drop : nullptr, stream)
               ? FA_OK
               : FA_ERR_CUDA;
}

fa_status fa_backward_deterministic(const void* Q, const void* K, const void* V, const void* O,
                                    const void* dO, const float* LSE, void* dQ, void* dK,
                                    void* dV, void* workspace, size_t workspace_bytes,
                                    const int* seqlens, int B, int H, int H_kv, int N, int d,
                                    float scale, int causal, float dropout_p,
                                    unsigned long long seed, unsigned int offset,
                                    cudaStream_t stream) {
    DropoutParams drop;
    bool on = false;
    fa_status st = make_dropout(dropout_p, seed, offset, &drop, &on);
    if (st != FA_OK) return st;
    if (!Q || !K || !V || !O || !dO || !LSE || !dQ || !dK || !dV || !workspace)
        return FA_ERR_INVALID_ARG;
    if (seqlens && (reinterpret_cast<uintptr_t>(seqlens) & 3u)) return FA_ERR_INVALID_ARG;
    const void* ptrs[] = {Q, K, V, O, dO, LSE, dQ, dK, dV, workspace};
    for (const void* p : ptrs)
        if (!aligned16(p)) return FA_ERR_INVALID_ARG;
    if ((st = check_shape(B, H, N, d, scale)) != FA_OK) return st;
    if ((st = check_heads(H, H_kv)) != FA_OK) return st;
    if (workspace_bytes < bwd_workspace_bytes(B, H, N, d)) return FA_ERR_INVALID_ARG;
    DeviceState* ds = current_device(&st);
    if (!ds) return st;
    if (!ensure_bwd_attributes(ds, d, on)) return FA_ERR_CUDA;
    return bwd_launch(Q, K, V, O, dO, LSE, dQ, dK, dV, workspace, B, H, H_kv, N, d, seqlens,
                      scale, causal, ds->err, on ? &drop : nullptr, stream, true)
               ? FA_OK
               : FA_ERR_CUDA;
}

fa_status fa_backward_varlen(const void* Q, const void* K, const void* V, const void* O,
                             const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                             void* workspace, size_t workspace_bytes, const int* seqlens, int B,
                             int H, int H_kv, int N, int d, float scale, int causal,
                             cudaStream_t stream) {
    if (!Q || !K || !V || !O || !dO || !LSE || !dQ || !dK || !dV || !workspace)
        return FA_ERR_INVALID_ARG;
    if (seqlens && (reinterpret_cast<uintptr_t>(seqlens) & 3u)) return FA_ERR_INVALID_ARG;
    const void* ptrs[] = {Q, K, V, O, dO, LSE, dQ, dK, dV, workspace};
    for (const void* p : ptrs)
        if (!aligned16(p)) return FA_ERR_INVALID_ARG;
    fa_status st = check_shape(B, H, N, d, scale);
    if (st != FA_OK) return st;
    if ((st = check_heads(H, H_kv)) != FA_OK) return st;
    if (workspace_bytes < bwd_workspace_bytes(B, H, N, d)) return FA_ERR_INVALID_ARG;
    DeviceState* ds = current_device(&st);
    if (!ds) return st;
    if (!ensure_bwd_attributes(ds, d, false)) return FA_ERR_CUDA;
    return bwd_launch(Q, K, V, O, dO, LSE, dQ, dK, dV, workspace, B, H, H_kv, N, d, seqlens,
                      scale, causal, ds->err, nullptr, stream)
               ? FA_OK
               : FA_ERR_CUDA;
}

fa_status fa_backward_gqa(const void* Q, const void* K, const void* V, const void* O,
                          const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                          void* workspace, size_t workspace_bytes, int B, int H, int H_kv, int N,
                          int d, float scale, int causal, cudaStream_t stream) {
    return fa_backward_varlen(Q, K, V, O, dO, LSE, dQ, dK, dV, workspace, workspace_bytes,
                              nullptr, B, H, H_kv, N, d, scale, causal, stream);
}

fa_status fa_backward(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                      const float* LSE, void* dQ, void* dK, void* dV, void* workspace,
                      size_t workspace_bytes, int B, int H, int N, int d, float scale,
                      int causal, cudaStream_t stream) {
    return fa_backward_gqa(Q, K, V, O, dO, LSE, dQ, dK, dV, workspace, workspace_bytes, B, H, H,
                           N, d, scale, causal, stream);
}

fa_status fa_check_device_error(cudaStream_t stream, unsigned int* site) {
    if (site) *site = 0;
    fa_status st;
    DeviceState* ds = current_device(&st);
    if (!ds) return st;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return FA_ERR_CUDA;
    uint32_t v = 0;
    if (cudaMemcpyFromSymbol(&v, g_err_word, sizeof(v)) != cudaSuccess) return FA_ERR_CUDA;
    if (v != 0) {
        const uint32_t zero = 0;
        if (cudaMemcpyToSymbol(g_err_word, &zero, sizeof(zero)) != cudaSuccess) return FA_ERR_CUDA;
    }
    if (site) *site = v;
    return v ? FA_ERR_TIMEOUT : FA_OK;
}

fa_status fa_selftest_bounded_wait(unsigned long long timeout_ns, cudaStream_t stream) {
    if (timeout_ns == 0 || timeout_ns > 1000000000ull) return FA_ERR_INVALID_ARG;
    fa_status st;
    DeviceState* ds = current_device(&st);
    if (!ds) return st;
    fa_selftest_wait_kernel<<<1, 64, 0, stream>>>(ds->err, timeout_ns, nullptr);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

const char* fa_status_str(fa_status s) {
    switch (s) {
        case FA_OK: return "ok";
        case FA_ERR_INVALID_ARG: return "invalid argument";
        case FA_ERR_UNSUPPORTED: return "unsupported shape or device (needs sm_100, d in {64,128})";
        case FA_ERR_CUDA: return "CUDA runtime error";
        case FA_ERR_TIMEOUT: return "device-side bounded wait expired";
    }
    return "unknown status";
}

int fa_version(void) { return 100; }

}  // extern "C"

// ---------------------------------------------------------------------------
// fa_backward_noalloc: the backward pass with its scratch in a fixed device
// array that lives inside this library.  For callers that must not allocate
// device memory themselves -- code running under a framework or engine whose
// allocator owns the whole device (a caching pool, a fixed memory budget) and
// does not allow raw cudaMalloc, or code on a latency-critical path that
// cannot take the device-wide synchronisation a cudaMalloc/cudaFree can
// cause.  Nothing here allocates: the array is reserved when the library's
// device code is loaded, on every GPU that loads it, and is released only when
// the process exits.
// ---------------------------------------------------------------------------
namespace fa {
namespace {

static __device__ __align__(256) unsigned char
    g_noalloc_scratch[FA_BACKWARD_NOALLOC_MAX_SCRATCH_BYTES];

struct NoallocDevice {
    bool ready = false;
    void* scratch = nullptr;  // device address of g_noalloc_scratch on this GPU
};
NoallocDevice g_noalloc[kMaxDevices];

}  // namespace
}  // namespace fa

extern "C" fa_status fa_backward_noalloc(const void* Q, const void* K, const void* V,
                                         const void* O, const void* dO, const float* LSE,
                                         void* dQ, void* dK, void* dV, int B, int H, int N,
                                         int d, float scale, int causal, cudaStream_t stream) {
    if (!Q || !K || !V || !O || !dO || !LSE || !dQ || !dK || !dV) return FA_ERR_INVALID_ARG;
    const void* ptrs[] = {Q, K, V, O, dO, LSE, dQ, dK, dV};
    for (const void* p : ptrs)
        if (!aligned16(p)) return FA_ERR_INVALID_ARG;
    fa_status st = check_shape(B, H, N, d, scale);
    if (st != FA_OK) return st;
    // The whole workspace must fit in the fixed array.
    if (bwd_workspace_bytes(B, H, N, d) > FA_BACKWARD_NOALLOC_MAX_SCRATCH_BYTES)
        return FA_ERR_UNSUPPORTED;
    DeviceState* ds = current_device(&st);
    if (!ds) return st;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        NoallocDevice& nd = g_noalloc[dev];
        if (!nd.ready) {
            // Once per device, with that device current: in host code the
            // array's name only stands in for it, so fetch its real address.
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
                return FA_ERR_CUDA;
            nd.scratch = p;
            nd.ready = true;
        }
        scratch = nd.scratch;
    }
    if (!ensure_bwd_attributes(ds, d, false)) return FA_ERR_CUDA;
    // Same three kernels as fa_backward; the preprocess kernel rewrites every
    // byte of the scratch the later kernels read (D, LSE and the zeroed fp32
    // dQ accumulator), so what an earlier call left there does not matter.
    return bwd_launch(Q, K, V, O, dO, LSE, dQ, dK, dV, scratch, B, H, H, N, d, nullptr, scale,
                      causal, ds->err, nullptr, stream)
               ? FA_OK
               : FA_ERR_CUDA;
}
