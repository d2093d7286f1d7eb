// C-ABI entry points of libdust: argument validation, workspace checks, the per-device error
// word, TMA descriptor encoding, and the generator test export.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>
#include <vector>

#include "dust_device.cuh"
#include "dust_internal.h"

namespace dust {

__device__ ErrorWord g_error_word;

namespace {

constexpr int kMaxDevices = 64;

int current_device() {
    int dev = 0;
    cudaGetDevice(&dev);
    return dev;
}

__global__ void philox_debug_kernel(const uint32_t* __restrict__ ctr, int64_t n, NoiseKey key,
                                    uint32_t* words, float* normals) {
    for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < n;
         j += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const uint4 c = reinterpret_cast<const uint4*>(ctr)[j];
        const U4 w = philox4x32_10(c.x, c.y, c.z, c.w, key);
        if (words) reinterpret_cast<uint4*>(words)[j] = make_uint4(w.x, w.y, w.z, w.w);
        if (normals) {
            const F4 z = normal_quad(c.x, c.y, c.z, c.w, key);
            reinterpret_cast<float4*>(normals)[j] = make_float4(z.x, z.y, z.z, z.w);
        }
    }
}

// Generator throughput probe: thread g sums the normals of the quads (j, g, 0, layer) for
// j < n_quads.  Generation plus one add per normal and nothing else, so its rate is the
// ceiling that the noise kernels' generator reaches on the device.
__global__ void __launch_bounds__(256) normal_sum_kernel(const __grid_constant__ NoiseKey key,
                                                         int64_t n, int32_t n_quads, float* out) {
    for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < n;
         g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const uint32_t t = key.token_offset + static_cast<uint32_t>(g);
        const PhiloxRun run = philox_run_over_word0(t, key.draw_offset, key.layer, key);
        F2 acc{0.f, 0.f};  // lanes: the quad's two polar pairs
#pragma unroll 2
        for (int32_t j = 0; j < n_quads; ++j) {
            const PolarPairs z =
                box_muller_pairs(philox_word0(key.quad_offset + static_cast<uint32_t>(j), run, key));
            acc = fma2(z.nq, add2(z.c, z.s), acc);
        }
        out[g] = kKappa * (acc.x + acc.y);
    }
}

// Philox-only throughput probe: thread g XORs together the words of the blocks
// (j, g, draw, layer) for j < n_blocks.  The generator's integer part alone (its widening
// multiplies and XORs), so its rate shows what the multiply pipe allows the noise kernels.
__global__ void __launch_bounds__(256) word_sum_kernel(const __grid_constant__ NoiseKey key,
                                                       int64_t n, int32_t n_blocks,
                                                       uint32_t* out) {
    for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < n;
         g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const uint32_t t = key.token_offset + static_cast<uint32_t>(g);
        const PhiloxRun run = philox_run_over_word0(t, key.draw_offset, key.layer, key);
        uint32_t acc = 0;
#pragma unroll 2
        for (int32_t j = 0; j < n_blocks; ++j) {
            const U4 w = philox_word0(key.quad_offset + static_cast<uint32_t>(j), run, key);
            acc ^= w.x ^ w.y ^ w.z ^ w.w;
        }
        out[g] = acc;
    }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

}  // namespace

void* current_context() {
    using CtxGetCurrent = CUresult (*)(CUcontext*);
    static CtxGetCurrent fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrent>(p);
    });
    CUcontext c = nullptr;
    if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
    return c;
}

ErrorWord* device_error_word() {
    static SymbolAddressCache cache;
    return static_cast<ErrorWord*>(cache.get([] {
        void* p = nullptr;
        return cudaGetSymbolAddress(&p, g_error_word) == cudaSuccess ? p : nullptr;
    }));
}

int num_sms() {
    // the count never changes for a device; several host threads may fill an entry at once
    // and store the same value (atomic, so that is not a data race)
    static std::atomic<int> cache[kMaxDevices];
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return 148;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (!n) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                       uint32_t box_rows, uint32_t box_cols) {
    auto fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_f32_2d_sw128(CUtensorMap* map, const float* base, uint64_t rows, uint64_t cols,
                            uint64_t ld, uint32_t box_rows) {
    auto fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {ld * 4};
    cuuint32_t box[2] = {32, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {
struct ProfRecord {
    const char* name;
    cudaEvent_t start, stop;
};
std::vector<ProfRecord> g_prof;       // completed records
std::vector<cudaEvent_t> g_prof_pool;  // free events
int g_prof_capacity = 0;
bool g_prof_on = false;
cudaEvent_t g_prof_open = nullptr;

cudaEvent_t prof_event() {
    if (!g_prof_pool.empty()) {
        cudaEvent_t e = g_prof_pool.back();
        g_prof_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}
}  // namespace

void prof_begin(cudaStream_t s) {
    if (!g_prof_on || static_cast<int>(g_prof.size()) >= g_prof_capacity) return;
    g_prof_open = prof_event();
    if (g_prof_open) cudaEventRecord(g_prof_open, s);
}

void prof_end(cudaStream_t s, const char* name) {
    if (!g_prof_on || !g_prof_open) return;
    cudaEvent_t stop = prof_event();
    if (stop) {
        cudaEventRecord(stop, s);
        g_prof.push_back(ProfRecord{name, g_prof_open, stop});
    } else {
        g_prof_pool.push_back(g_prof_open);
    }
    g_prof_open = nullptr;
}

dust_status philox_debug_launch(const uint32_t* ctr, int64_t n, NoiseKey key, uint32_t* words,
                                float* normals, cudaStream_t s) {
    if (n == 0) return DUST_OK;
    const unsigned blocks = static_cast<unsigned>(std::min<int64_t>((n + 255) / 256, static_cast<int64_t>(num_sms()) * 8));
    prof_begin(s);
    philox_debug_kernel<<<blocks, 256, 0, s>>>(ctr, n, key, words, normals);
    prof_end(s, "philox_debug");
    return cudaGetLastError() == cudaSuccess ? DUST_OK : DUST_ERR_CUDA;
}

dust_status normal_sum_launch(NoiseKey key, int64_t n, int32_t n_quads, float* out,
                              cudaStream_t s) {
    if (n == 0) return DUST_OK;
    const unsigned blocks = static_cast<unsigned>(std::min<int64_t>((n + 255) / 256, static_cast<int64_t>(num_sms()) * 8));
    prof_begin(s);
    normal_sum_kernel<<<blocks, 256, 0, s>>>(key, n, n_quads, out);
    prof_end(s, "normal_sum_probe");
    return cudaGetLastError() == cudaSuccess ? DUST_OK : DUST_ERR_CUDA;
}

dust_status word_sum_launch(NoiseKey key, int64_t n, int32_t n_blocks, uint32_t* out,
                            cudaStream_t s) {
    if (n == 0) return DUST_OK;
    const unsigned blocks = static_cast<unsigned>(std::min<int64_t>((n + 255) / 256, static_cast<int64_t>(num_sms()) * 8));
    prof_begin(s);
    word_sum_kernel<<<blocks, 256, 0, s>>>(key, n, n_blocks, out);
    prof_end(s, "word_sum_probe");
    return cudaGetLastError() == cudaSuccess ? DUST_OK : DUST_ERR_CUDA;
}

}  // namespace dust

using namespace dust;

namespace {

bool valid_dtype(dust_dtype dt) { return dt == DUST_F32 || dt == DUST_BF16; }

dust_status check_layer(const void* x, dust_dtype dt, int64_t N, int32_t d_in, int32_t d_out) {
    if (!valid_dtype(dt) || !x || N < 1 || d_in < 1 || d_out < 1) return DUST_ERR_INVALID_ARG;
    if (!aligned16(x)) return DUST_ERR_INVALID_ARG;
    if (N > 0xFFFFFFFFLL) return DUST_ERR_UNSUPPORTED;  // token index is one counter word
    if (dt == DUST_BF16 && (d_in % 16 != 0 || d_out % 16 != 0)) return DUST_ERR_UNSUPPORTED;
    if (dt == DUST_F32 && d_out % 4 != 0) return DUST_ERR_UNSUPPORTED;
    return DUST_OK;
}

dust_status check_ws(void* ws, size_t have, size_t need) {
    if (need == 0) return DUST_OK;
    if (!ws || !aligned256(ws) || have < need) return DUST_ERR_WORKSPACE;
    return DUST_OK;
}

}  // namespace

extern "C" {

const char* dust_status_string(dust_status s) {
    switch (s) {
        case DUST_OK: return "DUST_OK";
        case DUST_ERR_INVALID_ARG: return "DUST_ERR_INVALID_ARG";
        case DUST_ERR_UNSUPPORTED: return "DUST_ERR_UNSUPPORTED";
        case DUST_ERR_CUDA: return "DUST_ERR_CUDA";
        case DUST_ERR_TIMEOUT: return "DUST_ERR_TIMEOUT";
        case DUST_ERR_WORKSPACE: return "DUST_ERR_WORKSPACE";
    }
    return "DUST_ERR_UNKNOWN";
}

size_t dust_workspace_size(dust_op op, dust_dtype dt, int64_t N, int32_t d_in, int32_t d_out,
                           int32_t K) {
    if (N < 1 || K < 0) return 0;
    switch (op) {
        case DUST_OP_NOISY_LINEAR_FWD: return fwd_workspace_bytes(dt, N, d_out, K);
        case DUST_OP_CREDIT: return credit_workspace_bytes(N, K);
        case DUST_OP_WEIGHT_GRAD: return wgrad_workspace_bytes(dt, N, d_in, d_out);
        case DUST_OP_LOGITS_CE: return lmhead_workspace_bytes(N, d_out, K);
        case DUST_OP_SPSA_PROBE: return spsa_workspace_bytes(N, d_in, d_out, K);
    }
    return 0;
}

dust_status dust_noisy_logits_ce(const void* z, int64_t ld_z, dust_dtype dt, const int32_t* y,
                                 int64_t N, int32_t V, int32_t v0, int32_t S, int32_t K,
                                 float sigma, dust_noise_key key, float* dloss, int64_t ld_dloss,
                                 void* workspace, size_t ws_bytes, void* stream) {
    if (!valid_dtype(dt) || !z || !y || !dloss || N < 1 || V < 1 || K < 1 || ld_z < V ||
        ld_dloss < N)
        return DUST_ERR_INVALID_ARG;
    if (v0 < 0 || S < 0 || v0 % 4 != 0 || S % 4 != 0 || static_cast<int64_t>(v0) + S > V)
        return DUST_ERR_INVALID_ARG;
    if (!std::isfinite(sigma) || key.channel_offset != 0 || (reinterpret_cast<uintptr_t>(y) & 3u))
        return DUST_ERR_INVALID_ARG;
    if (N > 0xFFFFFFFFLL) return DUST_ERR_UNSUPPORTED;
    if (static_cast<uint64_t>(key.draw_offset) + static_cast<uint64_t>(K) > 0x100000000ull ||
        static_cast<uint64_t>(key.token_offset) + static_cast<uint64_t>(N) > 0x100000000ull)
        return DUST_ERR_INVALID_ARG;
    dust_status st = check_ws(workspace, ws_bytes, lmhead_workspace_bytes(N, S, K));
    if (st != DUST_OK) return st;
    return lmhead_launch(z, ld_z, dt, y, N, V, v0, S, K, sigma, make_key(key), dloss, ld_dloss,
                         workspace, static_cast<cudaStream_t>(stream));
}

dust_status dust_noisy_linear_fwd(const void* x, const void* W, const void* u, dust_dtype dt,
                                  int64_t N, int32_t d_in, int32_t d_out, int32_t K,
                                  float sigma, dust_noise_key key, float* dloss,
                                  int64_t ld_dloss, void* workspace, size_t ws_bytes,
                                  void* stream) {
    dust_status st = check_layer(x, dt, N, d_in, d_out);
    if (st != DUST_OK) return st;
    if (!W || !u || !dloss || !aligned16(W) || !aligned16(u) || !aligned16(dloss))
        return DUST_ERR_INVALID_ARG;
    if (K < 1 || ld_dloss < N || !std::isfinite(sigma) || key.channel_offset % 4 != 0)
        return DUST_ERR_INVALID_ARG;
    if (static_cast<uint64_t>(key.draw_offset) + static_cast<uint64_t>(K) > 0x100000000ull ||
        static_cast<uint64_t>(key.token_offset) + static_cast<uint64_t>(N) > 0x100000000ull)
        return DUST_ERR_INVALID_ARG;
    st = check_ws(workspace, ws_bytes, fwd_workspace_bytes(dt, N, d_out, K));
    if (st != DUST_OK) return st;
    return fwd_launch(x, W, u, dt, N, d_in, d_out, K, sigma, make_key(key), dloss, ld_dloss,
                      workspace, static_cast<cudaStream_t>(stream));
}

dust_status dust_credit(const float* loss, int64_t ld_loss, int32_t K, int64_t N,
                        const int32_t* cu_seqlens, int32_t n_seq, float gamma, float* r,
                        int64_t ld_r, void* workspace, size_t ws_bytes, void* stream) {
    if (!loss || !r || !cu_seqlens || N < 1 || K < 2 || n_seq < 1 || ld_loss < N || ld_r < N)
        return DUST_ERR_INVALID_ARG;
    if (!(gamma >= 0.f && gamma <= 1.f)) return DUST_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0 || !aligned16(loss) || !aligned16(r))
        return DUST_ERR_INVALID_ARG;
    dust_status st = check_ws(workspace, ws_bytes, credit_workspace_bytes(N, K));
    if (st != DUST_OK) return st;
    return credit_launch(loss, ld_loss, K, N, cu_seqlens, n_seq, gamma, r, ld_r, workspace,
                         static_cast<cudaStream_t>(stream));
}

dust_status dust_noisy_linear_output(const void* x, const void* W, dust_dtype dt, int64_t N,
                                     int32_t d_in, int32_t d_out, int32_t K, float sigma,
                                     dust_noise_key key, void* y_out, dust_dtype out_dt,
                                     int64_t ld_out, void* stream) {
    dust_status st = check_layer(x, dt, N, d_in, d_out);
    if (st != DUST_OK) return st;
    if (!W || !y_out || !aligned16(W) || !aligned16(y_out) || K < 1 || ld_out < d_out ||
        !valid_dtype(out_dt) || !std::isfinite(sigma) || key.channel_offset % 4 != 0)
        return DUST_ERR_INVALID_ARG;
    if (ld_out % (out_dt == DUST_BF16 ? 8 : 4) != 0) return DUST_ERR_INVALID_ARG;
    if (static_cast<uint64_t>(key.draw_offset) + static_cast<uint64_t>(K) > 0x100000000ull ||
        static_cast<uint64_t>(key.token_offset) + static_cast<uint64_t>(N) > 0x100000000ull)
        return DUST_ERR_INVALID_ARG;
    if (dt != DUST_BF16 || N > 2147483647LL) return DUST_ERR_UNSUPPORTED;
    return noisy_output_launch(x, W, N, d_in, d_out, K, sigma, make_key(key), y_out,
                               out_dt == DUST_BF16 ? 1 : 0, ld_out,
                               static_cast<cudaStream_t>(stream));
}

dust_status dust_spsa_probe(const void* x, const void* W, const void* u, dust_dtype dt, int64_t N,
                            int32_t d_in, int32_t d_out, int32_t P, float eps,
                            dust_noise_key key, float* p, float* L_plus, float* L_minus,
                            void* workspace, size_t ws_bytes, void* stream) {
    if (!x || !W || !u || !p || N < 1 || d_in < 1 || d_out < 1 || P < 1 || !valid_dtype(dt))
        return DUST_ERR_INVALID_ARG;
    if (!(eps > 0.f) || !std::isfinite(eps) || key.token_offset != 0 || key.channel_offset != 0 ||
        key.layer_id >= 0x80000000u)
        return DUST_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(W) || !aligned16(u)) return DUST_ERR_INVALID_ARG;
    if (static_cast<uint64_t>(key.draw_offset) + static_cast<uint64_t>(P) > 0x100000000ull)
        return DUST_ERR_INVALID_ARG;
    if (dt != DUST_BF16 || d_in % 16 != 0 || d_out % 16 != 0 || N > 2147483647LL ||
        static_cast<int64_t>(P) * ((d_out + 255) / 256 * 256) > 2147483647LL)
        return DUST_ERR_UNSUPPORTED;
    dust_status st = check_ws(workspace, ws_bytes, spsa_workspace_bytes(N, d_in, d_out, P));
    if (st != DUST_OK) return st;
    return spsa_probe_launch(x, W, u, N, d_in, d_out, P, eps, make_key(key), p, L_plus, L_minus,
                             workspace, static_cast<cudaStream_t>(stream));
}

dust_status dust_spsa_estimate(const float* p, int32_t P, int32_t P_total, int32_t d_in,
                               int32_t d_out, dust_noise_key key, float* G, int accumulate,
                               void* stream) {
    if (!p || !G || P < 1 || P_total < P || d_in < 1 || d_out < 1 || d_in % 4 != 0 ||
        !aligned16(G) || key.token_offset != 0 || key.channel_offset != 0 ||
        key.layer_id >= 0x80000000u)
        return DUST_ERR_INVALID_ARG;
    if (static_cast<uint64_t>(key.draw_offset) + static_cast<uint64_t>(P) > 0x100000000ull)
        return DUST_ERR_INVALID_ARG;
    return spsa_estimate_launch(p, P, P_total, d_in, d_out, make_key(key), G, accumulate,
                                static_cast<cudaStream_t>(stream));
}

dust_status dust_attn_reward(const float* ghat, int64_t ld_g, const void* delta_o,
                             int64_t ld_delta_o, dust_dtype dt, int64_t N, int32_t d, int32_t K,
                             float* c, int64_t ld_c, void* stream) {
    if (!valid_dtype(dt) || !ghat || !delta_o || !c || N < 1 || d < 1 || K < 1 || ld_g < d ||
        ld_delta_o < d || ld_c < N)
        return DUST_ERR_INVALID_ARG;
    const int E = dt == DUST_BF16 ? 8 : 4;  // elements per 16 bytes
    if (!aligned16(ghat) || !aligned16(delta_o) || ld_g % 4 != 0 || ld_delta_o % E != 0)
        return DUST_ERR_INVALID_ARG;
    if (d % E != 0 || d > 6144) return DUST_ERR_UNSUPPORTED;
    return attn_reward_launch(ghat, ld_g, delta_o, ld_delta_o, dt, N, d, K, c, ld_c,
                              static_cast<cudaStream_t>(stream));
}

dust_status dust_discounted_credit(const float* c, int64_t ld_c, int32_t K, int64_t N,
                                   const int32_t* cu_seqlens, int32_t n_seq, float gamma,
                                   float* r, int64_t ld_r, void* workspace, size_t ws_bytes,
                                   void* stream) {
    if (!c || !r || !cu_seqlens || N < 1 || K < 1 || n_seq < 1 || ld_c < N || ld_r < N)
        return DUST_ERR_INVALID_ARG;
    if (!(gamma >= 0.f && gamma <= 1.f)) return DUST_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0 || !aligned16(c) || !aligned16(r))
        return DUST_ERR_INVALID_ARG;
    dust_status st = check_ws(workspace, ws_bytes, credit_workspace_bytes(N, K));
    if (st != DUST_OK) return st;
    return credit_launch(c, ld_c, K, N, cu_seqlens, n_seq, gamma, r, ld_r, workspace,
                         static_cast<cudaStream_t>(stream), 0);
}

dust_status dust_weight_grad(const float* r, int64_t ld_r, const void* x, dust_dtype dt,
                             int64_t N, int32_t d_in, int32_t d_out, int32_t K_chunk,
                             int32_t K_total, float sigma, dust_noise_key key, float* G_W,
                             int accumulate, float* g_out, int32_t g_terms, void* workspace,
                             size_t ws_bytes, void* stream) {
    dust_status st = check_layer(x, dt, N, d_in, d_out);
    if (st != DUST_OK) return st;
    if (!r || !G_W || !aligned16(G_W) || (g_out && !aligned16(g_out))) return DUST_ERR_INVALID_ARG;
    if (g_terms != 1 && g_terms != 2) return DUST_ERR_INVALID_ARG;
    if (2 * N > 2147483647LL) return DUST_ERR_UNSUPPORTED;  // operand row index is 32-bit
    if (K_chunk < 1 || K_total < K_chunk || ld_r < N || key.channel_offset % 4 != 0)
        return DUST_ERR_INVALID_ARG;
    if (!(sigma > 0.f) || !std::isfinite(sigma)) return DUST_ERR_INVALID_ARG;
    if (static_cast<uint64_t>(key.draw_offset) + static_cast<uint64_t>(K_chunk) > 0x100000000ull ||
        static_cast<uint64_t>(key.token_offset) + static_cast<uint64_t>(N) > 0x100000000ull)
        return DUST_ERR_INVALID_ARG;
    size_t need = wgrad_workspace_bytes(dt, N, d_in, d_out);
    if (dt == DUST_F32 && g_out) need = 0;
    st = check_ws(workspace, ws_bytes, need);
    if (st != DUST_OK) return st;
    return wgrad_launch(r, ld_r, x, dt, N, d_in, d_out, K_chunk, K_total, sigma, make_key(key),
                        G_W, accumulate, g_out, g_terms, workspace,
                        static_cast<cudaStream_t>(stream));
}

dust_status dust_optimizer_step(const dust_opt_params* opt, const float* G, float* W,
                                void* W_bf16, float* m, float* v, int64_t n, void* stream) {
    OptParams o;
    if (!make_opt(opt, &o) || n < 0) return DUST_ERR_INVALID_ARG;
    if (n > 0 && (!G || !W || !m || (o.kind == DUST_OPT_ADAM && !v))) return DUST_ERR_INVALID_ARG;
    if (!aligned16(G) || !aligned16(W) || !aligned16(m) || (v && !aligned16(v)) ||
        (W_bf16 && (reinterpret_cast<uintptr_t>(W_bf16) & 7u) != 0))
        return DUST_ERR_INVALID_ARG;
    return opt_launch(o, G, OptTargets{W, W_bf16, m, v}, n, static_cast<cudaStream_t>(stream));
}

dust_status dust_weight_grad_step(const float* r, int64_t ld_r, const void* x, dust_dtype dt,
                                  int64_t N, int32_t d_in, int32_t d_out, int32_t K_chunk,
                                  int32_t K_total, float sigma, dust_noise_key key, float* G_W,
                                  int accumulate, float* g_out, int32_t g_terms,
                                  const dust_opt_params* opt, float* W, void* W_bf16, float* m,
                                  float* v, void* workspace, size_t ws_bytes, void* stream) {
    dust_status st = check_layer(x, dt, N, d_in, d_out);
    if (st != DUST_OK) return st;
    if (dt != DUST_BF16) return DUST_ERR_UNSUPPORTED;
    if (g_terms != 1 && g_terms != 2) return DUST_ERR_INVALID_ARG;
    if (2 * N > 2147483647LL) return DUST_ERR_UNSUPPORTED;
    OptParams o;
    if (!make_opt(opt, &o)) return DUST_ERR_INVALID_ARG;
    if (!r || (G_W && !aligned16(G_W)) || (accumulate && !G_W) || (g_out && !aligned16(g_out)))
        return DUST_ERR_INVALID_ARG;
    if (!W || !m || (o.kind == DUST_OPT_ADAM && !v) || !aligned16(W) || !aligned16(m) ||
        (v && !aligned16(v)) || (W_bf16 && (reinterpret_cast<uintptr_t>(W_bf16) & 7u) != 0))
        return DUST_ERR_INVALID_ARG;
    if (K_chunk < 1 || K_total < K_chunk || ld_r < N || key.channel_offset % 4 != 0) return DUST_ERR_INVALID_ARG;
    if (!(sigma > 0.f) || !std::isfinite(sigma)) return DUST_ERR_INVALID_ARG;
    if (static_cast<uint64_t>(key.draw_offset) + static_cast<uint64_t>(K_chunk) > 0x100000000ull ||
        static_cast<uint64_t>(key.token_offset) + static_cast<uint64_t>(N) > 0x100000000ull)
        return DUST_ERR_INVALID_ARG;
    st = check_ws(workspace, ws_bytes, wgrad_workspace_bytes(dt, N, d_in, d_out));
    if (st != DUST_OK) return st;
    const OptTargets t{W, W_bf16, m, v};
    return wgrad_launch(r, ld_r, x, dt, N, d_in, d_out, K_chunk, K_total, sigma, make_key(key),
                        G_W, accumulate, g_out, g_terms, workspace,
                        static_cast<cudaStream_t>(stream), &o, &t);
}

dust_status dust_last_device_error(void* stream, int32_t* info) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DUST_ERR_CUDA;
    ErrorWord* ew = device_error_word();
    if (!ew) return DUST_ERR_CUDA;
    ErrorWord h{0, 0};
    if (cudaMemcpy(&h, ew, sizeof h, cudaMemcpyDeviceToHost) != cudaSuccess) return DUST_ERR_CUDA;
    if (h.code != 0) {
        const ErrorWord zero{0, 0};
        if (cudaMemcpy(ew, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess)
            return DUST_ERR_CUDA;
    }
    if (info) *info = h.info;
    return h.code == 0 ? DUST_OK : static_cast<dust_status>(h.code);
}

dust_status dust_debug_philox(const uint32_t* ctr, int64_t n, uint64_t seed, uint32_t* words,
                              float* normals, void* stream) {
    if (n < 0 || (n > 0 && !ctr)) return DUST_ERR_INVALID_ARG;
    if ((ctr && !aligned16(ctr)) || (words && !aligned16(words)) || (normals && !aligned16(normals)))
        return DUST_ERR_INVALID_ARG;
    dust_noise_key k{seed, 0, 0, 0, 0};
    return philox_debug_launch(ctr, n, make_key(k), words, normals,
                               static_cast<cudaStream_t>(stream));
}

dust_status dust_debug_normal_sum(dust_noise_key key, int64_t n, int32_t n_quads, float* out,
                                  void* stream) {
    if (n < 0 || n_quads < 0 || (n > 0 && !out) || key.channel_offset % 4 != 0)
        return DUST_ERR_INVALID_ARG;
    if (static_cast<uint64_t>(key.token_offset) + static_cast<uint64_t>(n) > 0x100000000ull ||
        static_cast<uint64_t>(key.channel_offset / 4) + static_cast<uint64_t>(n_quads) >
            0x100000000ull)
        return DUST_ERR_INVALID_ARG;
    return normal_sum_launch(make_key(key), n, n_quads, out, static_cast<cudaStream_t>(stream));
}

dust_status dust_debug_word_sum(dust_noise_key key, int64_t n, int32_t n_blocks, uint32_t* out,
                                void* stream) {
    if (n < 0 || n_blocks < 0 || (n > 0 && !out) || key.channel_offset % 4 != 0)
        return DUST_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(out) & 3u) != 0) return DUST_ERR_INVALID_ARG;
    if (static_cast<uint64_t>(key.token_offset) + static_cast<uint64_t>(n) > 0x100000000ull ||
        static_cast<uint64_t>(key.channel_offset / 4) + static_cast<uint64_t>(n_blocks) >
            0x100000000ull)
        return DUST_ERR_INVALID_ARG;
    return word_sum_launch(make_key(key), n, n_blocks, out, static_cast<cudaStream_t>(stream));
}

void dust_debug_credit_skip_publish(int32_t block) { g_credit_skip_publish = block; }

dust_status dust_debug_fwd_plan(int64_t N, int32_t K, int32_t n_layers, const int32_t* d_out,
                                int32_t sms, int32_t* persistent, int32_t* split) {
    if (N < 1 || K < 1 || n_layers < 1 || !d_out || sms < 1 || !persistent || !split)
        return DUST_ERR_INVALID_ARG;
    for (int32_t l = 0; l < n_layers; ++l)
        if (d_out[l] < 1) return DUST_ERR_INVALID_ARG;
    fwd_plan(d_out, n_layers, N, K, sms, persistent, split);
    return DUST_OK;
}

}  // extern "C"

namespace {

dust_status check_group(const dust_layer_desc* layers, int32_t n_layers, int64_t N, int32_t K,
                        dust_noise_key key, int step) {
    if (!layers || n_layers < 1 || N < 1 || K < 1 || key.channel_offset % 4 != 0) return DUST_ERR_INVALID_ARG;
    if (N > 0xFFFFFFFFLL) return DUST_ERR_UNSUPPORTED;
    if (static_cast<uint64_t>(key.draw_offset) + static_cast<uint64_t>(K) > 0x100000000ull ||
        static_cast<uint64_t>(key.token_offset) + static_cast<uint64_t>(N) > 0x100000000ull)
        return DUST_ERR_INVALID_ARG;
    for (int32_t l = 0; l < n_layers; ++l) {
        const dust_layer_desc& d = layers[l];
        if (d.reserved != 0 || d.d_in < 1 || d.d_out < 1) return DUST_ERR_INVALID_ARG;
        if (d.d_in % 16 != 0 || d.d_out % 16 != 0) return DUST_ERR_UNSUPPORTED;
        if (step == 0 && (!d.x || !d.W || !d.u || !d.dloss || !aligned16(d.x) || !aligned16(d.W) ||
                          !aligned16(d.u) || !aligned16(d.dloss) || d.ld_dloss < N))
            return DUST_ERR_INVALID_ARG;
        if (step == 1 && (!d.dloss || !d.r || !aligned16(d.dloss) || !aligned16(d.r) ||
                          d.ld_dloss < N || d.ld_r < N))
            return DUST_ERR_INVALID_ARG;
        if (step == 2 && (!d.x || !d.r || !d.G_W || !aligned16(d.x) || !aligned16(d.G_W) ||
                          (d.g_out && !aligned16(d.g_out)) || d.ld_r < N))
            return DUST_ERR_INVALID_ARG;
    }
    return DUST_OK;
}

std::vector<FwdLayerArgs> fwd_args(const dust_layer_desc* layers, int32_t n) {
    std::vector<FwdLayerArgs> v(n);
    for (int32_t l = 0; l < n; ++l)
        v[l] = FwdLayerArgs{layers[l].x, layers[l].W, layers[l].u, layers[l].d_in, layers[l].d_out,
                            layers[l].layer_id, layers[l].dloss, layers[l].ld_dloss};
    return v;
}

std::vector<WgradLayerArgs> wgrad_args(const dust_layer_desc* layers, int32_t n) {
    std::vector<WgradLayerArgs> v(n);
    for (int32_t l = 0; l < n; ++l)
        v[l] = WgradLayerArgs{layers[l].r, layers[l].ld_r, layers[l].x, layers[l].d_in,
                              layers[l].d_out, layers[l].layer_id, layers[l].G_W, layers[l].g_out};
    return v;
}

}  // namespace

extern "C" {

size_t dust_workspace_size_grouped(dust_op op, const dust_layer_desc* layers, int32_t n_layers,
                                   int64_t N, int32_t K) {
    if (!layers || n_layers < 1 || N < 1 || K < 0) return 0;
    switch (op) {
        case DUST_OP_NOISY_LINEAR_FWD: {
            auto a = fwd_args(layers, n_layers);
            return fwd_grouped_workspace_bytes(a.data(), n_layers, N, K);
        }
        case DUST_OP_CREDIT: return credit_grouped_workspace_bytes(n_layers, N, K);
        case DUST_OP_WEIGHT_GRAD: {
            auto a = wgrad_args(layers, n_layers);
            return wgrad_grouped_workspace_bytes(a.data(), n_layers, N);
        }
    }
    return 0;
}

dust_status dust_noisy_linear_fwd_grouped(const dust_layer_desc* layers, int32_t n_layers,
                                          int64_t N, int32_t K, float sigma, dust_noise_key key,
                                          void* workspace, size_t ws_bytes, void* stream) {
    dust_status st = check_group(layers, n_layers, N, K, key, 0);
    if (st != DUST_OK) return st;
    if (!std::isfinite(sigma)) return DUST_ERR_INVALID_ARG;
    auto a = fwd_args(layers, n_layers);
    st = check_ws(workspace, ws_bytes, fwd_grouped_workspace_bytes(a.data(), n_layers, N, K));
    if (st != DUST_OK) return st;
    return fwd_grouped_launch(a.data(), n_layers, N, K, sigma, make_key(key), workspace,
                              static_cast<cudaStream_t>(stream));
}

dust_status dust_credit_grouped(const dust_layer_desc* layers, int32_t n_layers, int32_t K,
                                int64_t N, const int32_t* cu_seqlens, int32_t n_seq, float gamma,
                                void* workspace, size_t ws_bytes, void* stream) {
    dust_noise_key none{0, 0, 0, 0, 0};
    dust_status st = check_group(layers, n_layers, N, K, none, 1);
    if (st != DUST_OK) return st;
    if (!cu_seqlens || n_seq < 1 || K < 2 || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0)
        return DUST_ERR_INVALID_ARG;
    if (!(gamma >= 0.f && gamma <= 1.f)) return DUST_ERR_INVALID_ARG;
    st = check_ws(workspace, ws_bytes, credit_grouped_workspace_bytes(n_layers, N, K));
    if (st != DUST_OK) return st;
    std::vector<CreditLayerArgs> a(n_layers);
    for (int32_t l = 0; l < n_layers; ++l)
        a[l] = CreditLayerArgs{layers[l].dloss, layers[l].ld_dloss, layers[l].r, layers[l].ld_r};
    return credit_grouped_launch(a.data(), n_layers, K, N, cu_seqlens, n_seq, gamma, workspace,
                                 static_cast<cudaStream_t>(stream));
}

dust_status dust_weight_grad_grouped(const dust_layer_desc* layers, int32_t n_layers, int64_t N,
                                     int32_t K_chunk, int32_t K_total, float sigma,
                                     dust_noise_key key, int accumulate, int32_t g_terms,
                                     void* workspace, size_t ws_bytes, void* stream) {
    dust_status st = check_group(layers, n_layers, N, K_chunk, key, 2);
    if (st != DUST_OK) return st;
    if (K_total < K_chunk || !(sigma > 0.f) || !std::isfinite(sigma)) return DUST_ERR_INVALID_ARG;
    if (g_terms != 1 && g_terms != 2) return DUST_ERR_INVALID_ARG;
    if (2 * N > 2147483647LL) return DUST_ERR_UNSUPPORTED;
    auto a = wgrad_args(layers, n_layers);
    st = check_ws(workspace, ws_bytes, wgrad_grouped_workspace_bytes(a.data(), n_layers, N));
    if (st != DUST_OK) return st;
    return wgrad_grouped_launch(a.data(), n_layers, N, K_chunk, K_total, sigma, make_key(key),
                                accumulate, g_terms, workspace, static_cast<cudaStream_t>(stream));
}

dust_status dust_profile_enable(int32_t capacity) {
    if (capacity < 0) return DUST_ERR_INVALID_ARG;
    g_prof_capacity = capacity;
    g_prof_on = capacity > 0;
    return DUST_OK;
}

void dust_profile_disable(void) { g_prof_on = false; }

int32_t dust_profile_read(const char** names, float* ms, int32_t max) {
    cudaDeviceSynchronize();
    int32_t n = 0;
    for (const ProfRecord& r : g_prof) {
        if (n < max) {
            float t = 0.f;
            cudaEventElapsedTime(&t, r.start, r.stop);
            if (names) names[n] = r.name;
            if (ms) ms[n] = t;
            ++n;
        }
        g_prof_pool.push_back(r.start);
        g_prof_pool.push_back(r.stop);
    }
    g_prof.clear();
    return n;
}

}  // extern "C"
