// Host-side interface between the C-ABI entry points (dust_api.cu) and the kernel launchers
// of each stage.  Arguments arrive already validated.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <mutex>

#include "../../include/dust.h"

namespace dust {

struct ErrorWord;

// Philox4x32-10 round keys: key word j of round r is key_j + r * W_j (Weyl sequence with the
// constants of Salmon et al. 2011).  Computed once on the host so that kernels read them from
// parameter space instead of recomputing them per thread.
constexpr uint32_t kPhiloxWeyl0 = 0x9E3779B9u;
constexpr uint32_t kPhiloxWeyl1 = 0xBB67AE85u;

struct NoiseKey {
    uint32_t k0, k1;        // Philox key words (seed lo32, seed hi32)
    uint32_t layer;         // fourth counter word
    uint32_t draw_offset;   // added to the draw index (third counter word)
    uint32_t token_offset;  // added to the token index (second counter word)
    uint32_t quad_offset;   // added to the channel-quad index (first counter word)
    uint32_t rk[20];        // round keys: rk[2r] = k0 + r W0, rk[2r+1] = k1 + r W1
};

inline NoiseKey make_key(const dust_noise_key& k) {
    NoiseKey n{static_cast<uint32_t>(k.seed & 0xffffffffu), static_cast<uint32_t>(k.seed >> 32),
               k.layer_id, k.draw_offset, k.token_offset, k.channel_offset / 4, {}};
    for (uint32_t r = 0; r < 10; ++r) {
        n.rk[2 * r] = n.k0 + r * kPhiloxWeyl0;
        n.rk[2 * r + 1] = n.k1 + r * kPhiloxWeyl1;
    }
    return n;
}

ErrorWord* device_error_word();  // of the current device
int num_sms();                   // of the current device

// The CUDA context current on the calling thread (driver handle), or nullptr.
void* current_context();

// Device address of a file-scope __device__ array, per device context.  Host code only holds
// a stand-in for such an array, so its device address is looked up (by `lookup`, which must
// call cudaGetSymbolAddress in the file that defines the array) once per device, with that
// device current, and kept.  The entry is looked up again if the device's context changed
// (after cudaDeviceReset the module is loaded again, possibly at another address).  Calls
// from several host threads are serialised by a mutex.
class SymbolAddressCache {
  public:
    template <class Lookup>
    void* get(Lookup lookup) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
        void* ctx = current_context();
        std::lock_guard<std::mutex> guard(mu_);
        int slot = -1;
        for (int i = 0; i < n_; ++i)
            if (e_[i].dev == dev) slot = i;
        if (slot >= 0 && ctx && e_[slot].ctx == ctx) return e_[slot].ptr;
        void* p = lookup();
        if (!p) return nullptr;
        if (slot < 0) {
            if (n_ == kMax) return p;  // not cached; still correct
            slot = n_++;
        }
        e_[slot] = Entry{dev, current_context(), p};
        return p;
    }

  private:
    static constexpr int kMax = 64;
    struct Entry {
        int dev;
        void* ctx;
        void* ptr;
    };
    std::mutex mu_;
    Entry e_[kMax] = {};
    int n_ = 0;
};

// Runs `set` (returning true on success) once per device context: a kernel's function
// attributes belong to the context, so after a context reset the next call sets them again.
// Thread-safe; a failed `set` is tried again on the next call.
class PerContextOnce {
  public:
    template <class Set>
    bool run(Set set) {
        return cache_.get([&]() -> void* {
                   return set() ? reinterpret_cast<void*>(static_cast<uintptr_t>(1)) : nullptr;
               }) != nullptr;
    }

  private:
    SymbolAddressCache cache_;
};

// Encodes a 2-D row-major bf16 tensor [rows, cols] for TMA with a (box_cols x box_rows) box
// and 128-byte swizzle.  Returns false if the driver rejects it.
bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                       uint32_t box_rows, uint32_t box_cols);

// Encodes a 2-D row-major fp32 tensor [rows, cols] with leading dimension ld (elements) for
// TMA with a (32 x box_rows) box and 128-byte swizzle: 32 floats make one 128-byte line.
bool make_tmap_f32_2d_sw128(CUtensorMap* map, const float* base, uint64_t rows, uint64_t cols,
                            uint64_t ld, uint32_t box_rows);

// ---- noisy linear forward (dust_fwd.cu)
struct FwdLayerArgs {
    const void* x;
    const void* W;
    const void* u;
    int32_t d_in, d_out;
    uint32_t layer_id;
    float* dloss;
    int64_t ld;
};
size_t fwd_grouped_workspace_bytes(const FwdLayerArgs* layers, int n, int64_t N, int32_t K);
dust_status fwd_grouped_launch(const FwdLayerArgs* layers, int n, int64_t N, int32_t K,
                               float sigma, NoiseKey key, void* ws, cudaStream_t s);
size_t fwd_workspace_bytes(dust_dtype dt, int64_t N, int32_t d_out, int32_t K);
// The bf16 forward's form (persistent or one tile per CTA) and tail split for layers of these
// widths on `sms` SMs (host only).
void fwd_plan(const int32_t* d_out, int n, int64_t N, int32_t K, int64_t sms, int32_t* persistent,
              int32_t* split);
dust_status fwd_launch(const void* x, const void* W, const void* u, dust_dtype dt, int64_t N,
                       int32_t d_in, int32_t d_out, int32_t K, float sigma, NoiseKey key,
                       float* dloss, int64_t ld, void* ws, cudaStream_t s);

// ---- LM head on cached logits (dust_lmhead.cu)
size_t lmhead_workspace_bytes(int64_t N, int32_t S, int32_t K);
dust_status lmhead_launch(const void* z, int64_t ld_z, dust_dtype dt, const int32_t* y, int64_t N,
                          int32_t V, int32_t v0, int32_t S, int32_t K, float sigma, NoiseKey key,
                          float* dloss, int64_t ld, void* ws, cudaStream_t s);

// ---- credit (dust_credit.cu)
size_t credit_workspace_bytes(int64_t N, int32_t K);
dust_status credit_launch(const float* loss, int64_t ld_loss, int32_t K, int64_t N,
                          const int32_t* cu, int32_t n_seq, float gamma, float* r, int64_t ld_r,
                          void* ws, cudaStream_t s, int centre = 1);

// ---- SPSA / MeZO weight-space probe (dust_spsa.cu)
size_t spsa_workspace_bytes(int64_t N, int32_t d_in, int32_t d_out, int32_t P);
dust_status spsa_probe_launch(const void* x, const void* W, const void* u, int64_t N, int32_t d_in,
                              int32_t d_out, int32_t P, float eps, NoiseKey key, float* p,
                              float* Lp, float* Lm, void* ws, cudaStream_t s);
dust_status noisy_output_launch(const void* x, const void* W, int64_t N, int32_t d_in,
                               int32_t d_out, int32_t K, float sigma, NoiseKey key, void* y_out,
                               int out_bf16, int64_t ld_out, cudaStream_t s);
dust_status spsa_estimate_launch(const float* p, int32_t P, int32_t P_total, int32_t d_in,
                                 int32_t d_out, NoiseKey key, float* G, int accumulate,
                                 cudaStream_t s);

// ---- attention-internal reward (dust_attn.cu)
dust_status attn_reward_launch(const float* ghat, int64_t ld_g, const void* dO, int64_t ld_dO,
                               dust_dtype dt, int64_t N, int32_t d, int32_t K, float* c,
                               int64_t ld_c, cudaStream_t s);
extern int g_credit_skip_publish;
struct CreditLayerArgs {
    const float* loss;
    int64_t ld_loss;
    float* r;
    int64_t ld_r;
};
size_t credit_grouped_workspace_bytes(int n_layers, int64_t N, int32_t K);
dust_status credit_grouped_launch(const CreditLayerArgs* layers, int n, int32_t K, int64_t N,
                                  const int32_t* cu, int32_t n_seq, float gamma, void* ws,
                                  cudaStream_t s);

// ---- optimizer step on the weight estimate (dust_opt.cu, and fused in dust_wgrad.cu)
struct OptParams {
    int kind;             // 0: none, DUST_OPT_SGD_MOMENTUM, DUST_OPT_ADAM
    float lr, lr_wd;      // learning rate; lr * decoupled weight decay
    float mu;             // SGD momentum
    float b1, omb1, b2, omb2, eps, c1, c2;  // Adam: betas, 1 - betas, eps, 1 - beta^t
};
struct OptTargets {
    float* W;      // fp32 master weights (updated in place)
    void* W_bf16;  // optional bf16 copy of the updated weights
    float* m;      // first moment / momentum
    float* v;      // second moment (Adam)
};
bool make_opt(const dust_opt_params* p, OptParams* o);
dust_status opt_launch(const OptParams& o, const float* G, const OptTargets& t, int64_t n,
                       cudaStream_t s);

// ---- weight estimate (dust_wgrad.cu)
struct WgradLayerArgs {
    const float* r;
    int64_t ld_r;
    const void* x;
    int32_t d_in, d_out;
    uint32_t layer_id;
    float* G_W;
    float* g_out;
};
size_t wgrad_grouped_workspace_bytes(const WgradLayerArgs* layers, int n, int64_t N);
// g_terms: 1 (g rounded once to bf16) or 2 (hi + lo bf16 terms) for the bf16 contraction.
dust_status wgrad_grouped_launch(const WgradLayerArgs* layers, int n, int64_t N, int32_t K_chunk,
                                 int32_t K_total, float sigma, NoiseKey key, int accumulate,
                                 int g_terms, void* ws, cudaStream_t s);
size_t wgrad_workspace_bytes(dust_dtype dt, int64_t N, int32_t d_in, int32_t d_out);
dust_status wgrad_launch(const float* r, int64_t ld_r, const void* x, dust_dtype dt, int64_t N,
                         int32_t d_in, int32_t d_out, int32_t K_chunk, int32_t K_total,
                         float sigma, NoiseKey key, float* G_W, int accumulate, float* g_out,
                         int g_terms, void* ws, cudaStream_t s, const OptParams* opt = nullptr,
                         const OptTargets* targets = nullptr);

// ---- generator test export (dust_api.cu)
dust_status philox_debug_launch(const uint32_t* ctr, int64_t n, NoiseKey key, uint32_t* words,
                                float* normals, cudaStream_t s);

// Profiling hooks around each kernel launch (no-ops unless dust_profile_enable was called).
void prof_begin(cudaStream_t s);
void prof_end(cudaStream_t s, const char* name);

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Division of 0 <= f by a divisor d >= 1 fixed at launch, without a 64-bit divide in the
// kernel: with M = floor((2^64 - 1) / d) + 1 = 2^64 / d + e, 0 <= e < 1, the high word of f M
// is floor(f / d + f e 2^-64), and f e 2^-64 < 1 / d whenever f d < 2^64, so it cannot carry
// past the next multiple of 1 / d.  (d = 1 needs M = 2^64 and is handled apart.)
inline uint64_t div_magic(int64_t d) {
    return d > 1 ? ~0ull / static_cast<uint64_t>(d) + 1 : 0;
}
#ifdef __CUDACC__
__device__ __forceinline__ int64_t div_by_magic(int64_t f, int64_t d, uint64_t magic) {
    return d == 1 ? f : static_cast<int64_t>(__umul64hi(static_cast<uint64_t>(f), magic));
}
#endif

}  // namespace dust
