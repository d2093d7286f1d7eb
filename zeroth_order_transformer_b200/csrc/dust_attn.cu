// Attention-internal reward (Dust review page, section "간섭(interference) 줄이기", second
// point): the perturbations of the attention's internal projections (Q, K, V, gate) barely
// show in the token loss, so draw i is rewarded at token s by the alignment of the
// output-error estimate at the attention output with the change the draw caused there,
//   c_s^(i) = -<ghat_s, delta_o_s^(i)>,
// which then takes the place of the centred loss in the credit equation.
//
// HBM-bound: every element of delta_o [K, N, d] is read once.  Each warp owns one token at a
// time: it stages ghat_t in its own slice of shared memory, then streams the token's row of
// delta_o for every draw with 16-byte streaming loads (two draws in flight), multiplies by
// ghat_t and reduces with shuffles in a fixed order (deterministic).  No block-wide barrier.
// A lane's 16-byte load covers E consecutive elements; ghat is staged lane-minor (element j of
// lane l's group at j * 32 + l within each 32 E block), so the warp's shared reads of one j are
// 32 consecutive words, free of bank conflicts.
#include <algorithm>

#include "dust_device.cuh"
#include "dust_internal.h"

namespace dust {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ void load16(const float* p, float* v) {
    const float4 a = __ldcs(reinterpret_cast<const float4*>(p));
    v[0] = a.x;
    v[1] = a.y;
    v[2] = a.z;
    v[3] = a.w;
}
__device__ __forceinline__ void load16(const __nv_bfloat16* p, float* v) {
    const uint4 a = __ldcs(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        v[2 * j] = __uint_as_float(w[j] << 16);
        v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ float warp_sum(float a) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
    return a;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) attn_reward_kernel(const float* __restrict__ ghat,
                                                               int64_t ld_g, const T* __restrict__ dO,
                                                               int64_t ld_dO, int64_t N, int d,
                                                               int K, float* __restrict__ c,
                                                               int64_t ld_c) {
    constexpr int E = 16 / sizeof(T);  // elements per 16-byte load
    extern __shared__ float4 sm4[];    // kWarps slices of d floats
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slice = (d + 32 * E - 1) / (32 * E) * (32 * E);  // whole lane-minor blocks
    float* gs = reinterpret_cast<float*>(sm4) + static_cast<size_t>(warp) * slice;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kWarps;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * kWarps + warp; t < N; t += stride) {
        __syncwarp();  // the previous token's readers are done with the slice
        for (int k = lane * 4; k < d; k += 32 * 4) {
            const float4 g = __ldg(reinterpret_cast<const float4*>(ghat + t * ld_g + k));
            const float gv[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int kk = k + q;  // element kk sits in lane (kk % (32 E)) / E, slot kk % E
                gs[kk / (32 * E) * (32 * E) + (kk % E) * 32 + (kk % (32 * E)) / E] = gv[q];
            }
        }
        __syncwarp();
        const int64_t draw_stride = N * ld_dO;
        const T* row = dO + t * ld_dO;
        int i = 0;
        for (; i + 1 < K; i += 2) {
            const T* r0 = row + static_cast<int64_t>(i) * draw_stride;
            const T* r1 = r0 + draw_stride;
            float a0 = 0.f, a1 = 0.f;
#pragma unroll 2
            for (int k = lane * E; k < d; k += 32 * E) {
                float v0[E], v1[E];
                load16(r0 + k, v0);
                load16(r1 + k, v1);
                const float* gl = gs + (k - lane * E) + lane;
#pragma unroll
                for (int j = 0; j < E; ++j) {
                    const float g = gl[j * 32];
                    a0 = fmaf(g, v0[j], a0);
                    a1 = fmaf(g, v1[j], a1);
                }
            }
            a0 = warp_sum(a0);
            a1 = warp_sum(a1);
            if (lane == 0) {
                c[static_cast<int64_t>(i) * ld_c + t] = -a0;
                c[static_cast<int64_t>(i + 1) * ld_c + t] = -a1;
            }
        }
        if (i < K) {
            const T* r0 = row + static_cast<int64_t>(i) * draw_stride;
            float a0 = 0.f;
            for (int k = lane * E; k < d; k += 32 * E) {
                float v0[E];
                load16(r0 + k, v0);
                const float* gl = gs + (k - lane * E) + lane;
#pragma unroll
                for (int j = 0; j < E; ++j) a0 = fmaf(gl[j * 32], v0[j], a0);
            }
            a0 = warp_sum(a0);
            if (lane == 0) c[static_cast<int64_t>(i) * ld_c + t] = -a0;
        }
    }
}

}  // namespace

dust_status attn_reward_launch(const float* ghat, int64_t ld_g, const void* dO, int64_t ld_dO,
                               dust_dtype dt, int64_t N, int32_t d, int32_t K, float* c,
                               int64_t ld_c, cudaStream_t s) {
    const int blk = dt == DUST_BF16 ? 256 : 128;  // 32 lanes x elements per 16-byte load
    const size_t smem = static_cast<size_t>(kWarps) * ((d + blk - 1) / blk * blk) * 4;
    const unsigned blocks = static_cast<unsigned>(
        std::min<int64_t>((N + kWarps - 1) / kWarps, static_cast<int64_t>(num_sms()) * 16));
    if (dt == DUST_BF16) {
        auto k = attn_reward_kernel<__nv_bfloat16>;
        if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem)) != cudaSuccess)
            return DUST_ERR_CUDA;
        prof_begin(s);
        k<<<blocks, kThreads, smem, s>>>(ghat, ld_g, static_cast<const __nv_bfloat16*>(dO), ld_dO,
                                         N, d, K, c, ld_c);
    } else {
        auto k = attn_reward_kernel<float>;
        if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem)) != cudaSuccess)
            return DUST_ERR_CUDA;
        prof_begin(s);
        k<<<blocks, kThreads, smem, s>>>(ghat, ld_g, static_cast<const float*>(dO), ld_dO, N, d,
                                         K, c, ld_c);
    }
    prof_end(s, "attn_reward");
    return cudaGetLastError() == cudaSuccess ? DUST_OK : DUST_ERR_CUDA;
}

}  // namespace dust
