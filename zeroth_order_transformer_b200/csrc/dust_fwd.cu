// Noisy linear forward with the per-draw loss change (Dust review page, section "신용 할당",
// noise equation y_t -> y_t + sigma a_t, with the quadratic readout l = 1/2 |y + sigma a - u|^2).
//
// bf16 layers: one tcgen05 kernel per 128-token x 256-channel tile.  TMA brings x and W tiles
// (128-byte swizzle, 2-stage ring) into shared memory, one thread issues tcgen05.mma into a
// 128 x 256 fp32 accumulator in tensor memory.  The epilogue turns the accumulator into
// s_e = sigma (y - u) in place, then every thread owns one token and walks every draw:
// it regenerates the normals of its 256 channels (never stored) and sums
//   sigma a e + sigma^2 a^2 / 2
// into a per-tile partial.  The last tile of each token block (an atomic ticket) adds the
// partials of all channel tiles in a fixed order, so the result is deterministic.
//
// fp32 layers: a SIMT kernel (one warp per token, one quad of channels per lane) and a
// partial-sum reduction kernel.
#include "dust_device.cuh"
#include "dust_internal.h"

namespace dust {
namespace {

constexpr int kBM = 128;  // tokens per tile
constexpr int kBN = 256;  // channels per tile
constexpr int kBK = 64;   // d_in per pipeline stage (128 bytes of bf16: one swizzle row)
constexpr int kStages = 2;
constexpr int kThreads = 384;  // 3 groups of 4 warps
constexpr int kGroups = kThreads / 128;
constexpr uint32_t kABytes = kBM * kBK * 2;
constexpr uint32_t kBBytes = kBN * kBK * 2;
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kSmemBytes = kStages * kStageBytes + 1024 + 256;
constexpr uint32_t kTmemCols = 256;

struct FwdParams {
    const __nv_bfloat16* u;
    float* partial;  // [2 n_tiles, K, N]: (channel tile, half) x draw x token
    float* dloss;    // [K, ld]
    int* counters;   // [m_tiles], zero on entry
    ErrorWord* ew;
    int64_t N;
    int64_t ld;
    int d_in, d_out, K, n_tiles;
    float sigma, half_sigma2;
    NoiseKey key;
};

__device__ __forceinline__ void unpack_bf16x8(const uint4& v, float* f) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 p = __bfloat1622float2(h[j]);
        f[2 * j] = p.x;
        f[2 * j + 1] = p.y;
    }
}

__global__ void __launch_bounds__(kThreads, 2)
    fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmw,
                    const FwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
    uint64_t* empty = full + kStages;
    uint64_t* acc_full = empty + kStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
    int* is_last = reinterpret_cast<int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int m_tile = blockIdx.x;
    const int n_tile = blockIdx.y;
    const int64_t m0 = static_cast<int64_t>(m_tile) * kBM;
    const int n0 = n_tile * kBN;
    const int nk = (p.d_in + kBK - 1) / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        *is_last = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 && lane == 0) {
        // TMA producer
        prefetch_tensormap(&tmx);
        prefetch_tensormap(&tmw);
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % kStages;
            if (kb >= kStages &&
                !mbar_wait_bounded(&empty[s], ((kb / kStages) - 1) & 1, p.ew, 101))
                break;
            uint8_t* a = smem + s * kStageBytes;
            mbar_arrive_expect_tx(&full[s], kStageBytes);
            tma_load_2d(a, &tmx, &full[s], kb * kBK, static_cast<int32_t>(m0));
            tma_load_2d(a + kABytes, &tmw, &full[s], kb * kBK, n0);
        }
    } else if (warp == 1 && lane == 0) {
        // MMA issuer: 4 MMAs of K = 16 per stage; operands K-major, 128-byte swizzle,
        // 8-row core groups 1024 bytes apart.
        constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, 0, 0);
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % kStages;
            if (!mbar_wait_bounded(&full[s], (kb / kStages) & 1, p.ew, 102)) break;
            tc_fence_after();
            const uint32_t a_addr = smem_u32(smem + s * kStageBytes);
            const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
                const uint64_t ad = sdesc_sw128(a_addr + kk * 32, 16, 1024);
                const uint64_t bd = sdesc_sw128(b_addr + kk * 32, 16, 1024);
                umma_bf16(tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
            }
            umma_commit(&empty[s]);
        }
        umma_commit(acc_full);
    }

    mbar_wait_bounded(acc_full, 0, p.ew, 103);
    __syncwarp();
    tc_fence_after();

    // ---------------- epilogue: every warp; TMEM lane quarter = warp % 4, and the kGroups
    // warps that share a lane quarter split the work (chunks in phase 1, draws in phase 2).
    const int lq = warp & 3;
    const int grp = warp >> 2;
    const int row = lq * 32 + lane;
    const int64_t t = m0 + row;
    const bool valid = t < p.N;
    const uint32_t trow = tmem + (static_cast<uint32_t>(lq * 32) << 16);
    const int nchunks = min(kBN, p.d_out - n0) / 16;

    // Phase 1: s_e = sigma (y - u), written back in place.
    for (int c = grp; c < nchunks; c += kGroups) {
        float v[16];
        tmem_ld16(trow + c * 16, v);
        tmem_wait_ld();
        if (valid) {
            const uint4* up =
                reinterpret_cast<const uint4*>(p.u + t * p.d_out + n0 + c * 16);
            float uf[16];
            unpack_bf16x8(__ldg(up), uf);
            unpack_bf16x8(__ldg(up + 1), uf + 8);
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = p.sigma * (v[j] - uf[j]);
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = 0.f;
        }
        tmem_st16(trow + c * 16, v);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // Phase 2: work units are (draw, half of the tile's channels), dealt round-robin to the
    // warp groups so that they finish together.  Per unit: regenerate the noise and sum the
    // loss change over the half's channels.  In polar form a pair (z, z') = -rho (cos, sin)
    // contributes sigma (z e + z' e') + sigma^2 / 2 (z^2 + z'^2)
    //           = -rho (cos s_e + sin s_e') + h x,   with x = rho^2 = -2 ln u.
    const uint32_t tg = p.key.token_offset + static_cast<uint32_t>(t);
    const uint32_t qbase = static_cast<uint32_t>(n0 >> 2);
    const float h = p.half_sigma2;
    const int half_chunks = (nchunks + 1) / 2;
    for (int unit = grp; unit < 2 * p.K; unit += kGroups) {
        const int i = unit >> 1;
        const int hf = unit & 1;
        const uint32_t di = p.key.draw_offset + static_cast<uint32_t>(i);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        const int c_end = hf ? nchunks : half_chunks;
        for (int c = hf ? half_chunks : 0; c < c_end; ++c) {
            float se[16];
            tmem_ld16(trow + c * 16, se);
            tmem_wait_ld();
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                const Polar4 z = normal_quad_polar(qbase + c * 4 + qq, tg, di, p.key.layer, p.key);
                const float l0 = fmaf(z.s0, se[4 * qq + 1], z.c0 * se[4 * qq + 0]);
                const float l1 = fmaf(z.s1, se[4 * qq + 3], z.c1 * se[4 * qq + 2]);
                acc[qq] = fmaf(-z.r0, l0, acc[qq]);
                acc[qq] = fmaf(-z.r1, l1, acc[qq]);
                acc[qq] = fmaf(h, z.x0 + z.x1, acc[qq]);
            }
        }
        if (valid)
            p.partial[((static_cast<int64_t>(n_tile) * 2 + hf) * p.K + i) * p.N + t] =
                (acc[0] + acc[1]) + (acc[2] + acc[3]);
    }

    // Release tensor memory early, then the last channel tile of this token block reduces.
    tc_fence_before();
    __threadfence();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
    if (threadIdx.x == 0) {
        const int old = atomicAdd(&p.counters[m_tile], 1);
        *is_last = (old == p.n_tiles - 1);
    }
    __syncthreads();
    if (*is_last) {
        __threadfence();
        for (int idx = threadIdx.x; idx < p.K * kBM; idx += kThreads) {
            const int i = idx / kBM;
            const int64_t tt = m0 + (idx % kBM);
            if (tt < p.N) {
                float s = 0.f;
                for (int pp = 0; pp < 2 * p.n_tiles; ++pp)
                    s += __ldcg(&p.partial[(static_cast<int64_t>(pp) * p.K + i) * p.N + tt]);
                p.dloss[static_cast<int64_t>(i) * p.ld + tt] = s;
            }
        }
        if (threadIdx.x == 0) p.counters[m_tile] = 0;
    }
}

// ------------------------------------------------------------------------------ fp32 path
constexpr int kF32Tokens = 8;    // tokens per block (one warp each)
constexpr int kF32Quads = 32;    // channel quads per block (one lane each)

struct FwdF32Params {
    const float* x;
    const float* W;
    const float* u;
    float* partial;  // [n_cb, K, N]
    int64_t N;
    int d_in, d_out, K;
    float sigma, half_sigma2;
    NoiseKey key;
};

__global__ void __launch_bounds__(256) fwd_f32_kernel(const FwdF32Params p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * kF32Tokens + warp;
    const int cb = blockIdx.y;
    const int q = cb * kF32Quads + lane;
    const int o0 = 4 * q;
    const bool tok_ok = t < p.N;
    float se[4] = {0.f, 0.f, 0.f, 0.f};
    bool ch_ok[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) ch_ok[j] = tok_ok && (o0 + j < p.d_out);
    if (tok_ok) {
        const float* xt = p.x + t * p.d_in;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (!ch_ok[j]) continue;
            const float* Wo = p.W + static_cast<int64_t>(o0 + j) * p.d_in;
            float acc = 0.f;
            for (int k = 0; k < p.d_in; ++k) acc = fmaf(Wo[k], xt[k], acc);
            se[j] = p.sigma * (acc - p.u[t * p.d_out + o0 + j]);
        }
    }
    const uint32_t tg = p.key.token_offset + static_cast<uint32_t>(t);
    for (int i = 0; i < p.K; ++i) {
        float acc = 0.f;
        if (ch_ok[0]) {
            const F4 z = normal_quad(static_cast<uint32_t>(q), tg,
                                     p.key.draw_offset + static_cast<uint32_t>(i), p.key.layer, p.key);
            const float zz[4] = {z.x, z.y, z.z, z.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (ch_ok[j]) acc = fmaf(zz[j], fmaf(p.half_sigma2, zz[j], se[j]), acc);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0 && tok_ok) p.partial[(static_cast<int64_t>(cb) * p.K + i) * p.N + t] = acc;
    }
}

__global__ void reduce_partials_kernel(const float* __restrict__ partial, int n_parts, int K,
                                       int64_t N, float* __restrict__ out, int64_t ld) {
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<int64_t>(K) * N) return;
    const int i = static_cast<int>(idx / N);
    const int64_t t = idx % N;
    float s = 0.f;
    for (int pp = 0; pp < n_parts; ++pp) s += partial[(static_cast<int64_t>(pp) * K + i) * N + t];
    out[static_cast<int64_t>(i) * ld + t] = s;
}

}  // namespace

size_t fwd_workspace_bytes(dust_dtype dt, int64_t N, int32_t d_out, int32_t K) {
    if (dt == DUST_BF16) {
        const int64_t n_tiles = (d_out + kBN - 1) / kBN;
        const int64_t m_tiles = (N + kBM - 1) / kBM;
        return align_up(static_cast<size_t>(2 * n_tiles * K * N) * 4, 256) +
               align_up(static_cast<size_t>(m_tiles) * 4, 256);
    }
    const int64_t n_cb = (d_out + 4 * kF32Quads - 1) / (4 * kF32Quads);
    return align_up(static_cast<size_t>(n_cb * K * N) * 4, 256);
}

dust_status fwd_launch(const void* x, const void* W, const void* u, dust_dtype dt, int64_t N,
                       int32_t d_in, int32_t d_out, int32_t K, float sigma, NoiseKey key,
                       float* dloss, int64_t ld, void* ws, cudaStream_t s) {
    if (dt == DUST_BF16) {
        const int n_tiles = (d_out + kBN - 1) / kBN;
        const int64_t m_tiles = (N + kBM - 1) / kBM;
        if (m_tiles > 2147483647LL) return DUST_ERR_UNSUPPORTED;
        CUtensorMap tmx, tmw;
        if (!make_tmap_bf16_2d(&tmx, x, static_cast<uint64_t>(N), d_in, kBM, kBK) ||
            !make_tmap_bf16_2d(&tmw, W, static_cast<uint64_t>(d_out), d_in, kBN, kBK))
            return DUST_ERR_CUDA;
        FwdParams p;
        p.u = static_cast<const __nv_bfloat16*>(u);
        p.partial = static_cast<float*>(ws);
        p.counters = reinterpret_cast<int*>(static_cast<char*>(ws) +
                                            align_up(static_cast<size_t>(2 * n_tiles) * K * N * 4, 256));
        p.dloss = dloss;
        p.ew = device_error_word();
        p.N = N;
        p.ld = ld;
        p.d_in = d_in;
        p.d_out = d_out;
        p.K = K;
        p.n_tiles = n_tiles;
        p.sigma = sigma;
        p.half_sigma2 = 0.5f * sigma * sigma;
        p.key = key;
        static bool attr_done[64] = {};
        int dev = 0;
        cudaGetDevice(&dev);
        if (dev >= 64 || !attr_done[dev]) {
            if (cudaFuncSetAttribute(fwd_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kSmemBytes) != cudaSuccess)
                return DUST_ERR_CUDA;
            if (dev < 64) attr_done[dev] = true;
        }
        if (cudaMemsetAsync(p.counters, 0, static_cast<size_t>(m_tiles) * 4, s) != cudaSuccess)
            return DUST_ERR_CUDA;
        dim3 grid(static_cast<unsigned>(m_tiles), static_cast<unsigned>(n_tiles));
        prof_begin(s);
        fwd_bf16_kernel<<<grid, kThreads, kSmemBytes, s>>>(tmx, tmw, p);
        prof_end(s, "fwd_bf16_noise_loss");
        return cudaGetLastError() == cudaSuccess ? DUST_OK : DUST_ERR_CUDA;
    }
    const int n_cb = (d_out + 4 * kF32Quads - 1) / (4 * kF32Quads);
    FwdF32Params p;
    p.x = static_cast<const float*>(x);
    p.W = static_cast<const float*>(W);
    p.u = static_cast<const float*>(u);
    p.partial = static_cast<float*>(ws);
    p.N = N;
    p.d_in = d_in;
    p.d_out = d_out;
    p.K = K;
    p.sigma = sigma;
    p.half_sigma2 = 0.5f * sigma * sigma;
    p.key = key;
    dim3 grid(static_cast<unsigned>((N + kF32Tokens - 1) / kF32Tokens), static_cast<unsigned>(n_cb));
    prof_begin(s);
    fwd_f32_kernel<<<grid, 256, 0, s>>>(p);
    prof_end(s, "fwd_f32_noise_loss");
    const int64_t total = static_cast<int64_t>(K) * N;
    prof_begin(s);
    reduce_partials_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, s>>>(
        p.partial, n_cb, K, N, dloss, ld);
    prof_end(s, "fwd_f32_reduce_partials");
    return cudaGetLastError() == cudaSuccess ? DUST_OK : DUST_ERR_CUDA;
}

}  // namespace dust
