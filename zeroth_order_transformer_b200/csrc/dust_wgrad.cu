// Output-error estimate and weight estimate (Dust review page, section "신용 할당":
// g_t = -(1/(K sigma)) sum_i r_t^(i) a_t^(i) and G_W = sum_t g_t x_t^T).
//
// Stage 1 (ghat_kernel): one thread per (token, channel quad) regenerates the quad's normals
// for every draw and accumulates the reward-weighted sum; g is written as bf16 (the tensor
// core operand) and optionally as fp32.  A grid-stride loop over (token, 128-quad block)
// units keeps every SM busy to the end.
// Stage 2 (gw_bf16_kernel): G_W = g^T x on the tensor cores.  Both operands are MN-major
// (tokens are the contraction index and the slow index of g [N, d_out] and x [N, d_in]):
// TMA loads 64-token x 64-element boxes with 128-byte swizzle, one thread issues
// tcgen05.mma (M = 128 output rows, N = 256 output columns, K = 16 tokens per instruction)
// into a TMEM accumulator.  Small outputs split the token range (split-K) and a fixed-order
// reduction adds the partials, so the result is deterministic.
// fp32 layers use a SIMT tiled contraction on the fp32 g.
#include <algorithm>

#include "dust_device.cuh"
#include "dust_internal.h"

namespace dust {
namespace {

// ------------------------------------------------------------------ stage 1: g
constexpr int kGThreads = 128;

struct GhatParams {
    const float* r;
    __nv_bfloat16* gb;  // [N, d_out] or null
    float* gf;          // [N, d_out] or null
    int64_t ld_r, N, units;
    int d_out, K, nqb;
    float scale;  // -1 / (K_total sigma)
    NoiseKey key;
};

__global__ void __launch_bounds__(kGThreads) ghat_kernel(const GhatParams p) {
    const int nq = p.d_out >> 2;
    for (int64_t u = blockIdx.x; u < p.units; u += gridDim.x) {
        const int64_t t = u / p.nqb;
        const int q = static_cast<int>(u % p.nqb) * kGThreads + threadIdx.x;
        if (q >= nq) continue;
        const uint32_t tg = p.key.token_offset + static_cast<uint32_t>(t);
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        const float* rt = p.r + t;
        // unrolled so that independent Philox chains of consecutive draws interleave
#pragma unroll 2
        for (int i = 0; i < p.K; ++i) {
            const float ri = __ldg(rt + static_cast<int64_t>(i) * p.ld_r);
            const Polar4 z = normal_quad_polar(static_cast<uint32_t>(q), tg,
                                               p.key.draw_offset + static_cast<uint32_t>(i),
                                               p.key.layer, p.key);
            // r a = -(r rho) (cos, sin) per pair
            const float rr0 = ri * z.r0;
            const float rr1 = ri * z.r1;
            a0 = fmaf(-rr0, z.c0, a0);
            a1 = fmaf(-rr0, z.s0, a1);
            a2 = fmaf(-rr1, z.c1, a2);
            a3 = fmaf(-rr1, z.s1, a3);
        }
        a0 *= p.scale;
        a1 *= p.scale;
        a2 *= p.scale;
        a3 *= p.scale;
        const int64_t off = t * p.d_out + 4 * q;
        if (p.gb) {
            __nv_bfloat162 lo = __floats2bfloat162_rn(a0, a1);
            __nv_bfloat162 hi = __floats2bfloat162_rn(a2, a3);
            uint2 v;
            v.x = *reinterpret_cast<uint32_t*>(&lo);
            v.y = *reinterpret_cast<uint32_t*>(&hi);
            *reinterpret_cast<uint2*>(p.gb + off) = v;
        }
        if (p.gf) *reinterpret_cast<float4*>(p.gf + off) = make_float4(a0, a1, a2, a3);
    }
}

// ------------------------------------------------------------------ stage 2: G_W (bf16)
constexpr int kGM = 128;  // output rows (o) per tile
constexpr int kGN = 256;  // output columns (k) per tile
constexpr int kGK = 64;   // tokens per stage
constexpr int kGStages = 4;
constexpr int kGWThreads = 128;
constexpr uint32_t kBox = 64 * 64 * 2;  // one 64-token x 64-element box
constexpr uint32_t kGABytes = kGM / 64 * kBox;
constexpr uint32_t kGBBytes = kGN / 64 * kBox;
constexpr uint32_t kGStageBytes = kGABytes + kGBBytes;
constexpr uint32_t kGSmem = kGStages * kGStageBytes + 1024 + 256;
constexpr uint32_t kGTmemCols = 256;

struct GwParams {
    float* out;  // G_W (split == 1) or partial [S, d_out, d_in]
    ErrorWord* ew;
    int64_t N, tokens_per_split;
    int d_in, d_out, accumulate;
};

__global__ void __launch_bounds__(kGWThreads, 1)
    gw_bf16_kernel(const __grid_constant__ CUtensorMap tmg, const __grid_constant__ CUtensorMap tmx,
                   const GwParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGStages * kGStageBytes);
    uint64_t* empty = full + kGStages;
    uint64_t* acc_full = empty + kGStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int o0 = blockIdx.x * kGM;
    const int k0 = blockIdx.y * kGN;
    const int split = blockIdx.z;
    const int64_t t_begin = static_cast<int64_t>(split) * p.tokens_per_split;
    const int64_t t_end = min(p.N, t_begin + p.tokens_per_split);
    const int nk = t_end > t_begin ? static_cast<int>((t_end - t_begin + kGK - 1) / kGK) : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kGTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmg);
        prefetch_tensormap(&tmx);
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % kGStages;
            if (kb >= kGStages &&
                !mbar_wait_bounded(&empty[s], ((kb / kGStages) - 1) & 1, p.ew, 201))
                break;
            uint8_t* a = smem + s * kGStageBytes;
            uint8_t* bsm = a + kGABytes;
            const int32_t tok = static_cast<int32_t>(t_begin + static_cast<int64_t>(kb) * kGK);
            mbar_arrive_expect_tx(&full[s], kGStageBytes);
#pragma unroll
            for (int j = 0; j < kGM / 64; ++j) tma_load_2d(a + j * kBox, &tmg, &full[s], o0 + 64 * j, tok);
#pragma unroll
            for (int j = 0; j < kGN / 64; ++j)
                tma_load_2d(bsm + j * kBox, &tmx, &full[s], k0 + 64 * j, tok);
        }
    } else if (warp == 1 && lane == 0) {
        // MN-major operands: 64-element (128-byte) rows, one row per token; 8-token core
        // groups 1024 bytes apart (SBO); successive 64-element column blocks one box apart
        // (LBO); 16 tokens per instruction = 2048 bytes.
        constexpr uint32_t idesc = idesc_bf16_f32(kGM, kGN, 1, 1);
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % kGStages;
            if (!mbar_wait_bounded(&full[s], (kb / kGStages) & 1, p.ew, 202)) break;
            tc_fence_after();
            const uint32_t a_addr = smem_u32(smem + s * kGStageBytes);
            const uint32_t b_addr = a_addr + kGABytes;
#pragma unroll
            for (int kk = 0; kk < kGK / 16; ++kk) {
                const uint64_t ad = sdesc_sw128(a_addr + kk * 2048, kBox, 1024);
                const uint64_t bd = sdesc_sw128(b_addr + kk * 2048, kBox, 1024);
                umma_bf16(tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
            }
            umma_commit(&empty[s]);
        }
        umma_commit(acc_full);
    }

    mbar_wait_bounded(acc_full, 0, p.ew, 203);
    __syncwarp();
    tc_fence_after();

    const int o = o0 + warp * 32 + lane;
    const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const int ncols = min(kGN, p.d_in - k0);
    float* dst = p.out + static_cast<int64_t>(split) * p.d_out * p.d_in;
    for (int c = 0; c < ncols / 16; ++c) {
        float v[16];
        tmem_ld16(trow + c * 16, v);
        tmem_wait_ld();
        if (nk == 0) {
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = 0.f;
        }
        if (o < p.d_out) {
            float4* d4 = reinterpret_cast<float4*>(dst + static_cast<int64_t>(o) * p.d_in + k0 + c * 16);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float4 w = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                if (p.accumulate) {
                    const float4 old = d4[j];
                    w.x += old.x;
                    w.y += old.y;
                    w.z += old.z;
                    w.w += old.w;
                }
                d4[j] = w;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, kGTmemCols);
}

__global__ void splitk_reduce_kernel(const float4* __restrict__ part, int S, int64_t n4,
                                     float4* __restrict__ out, int accumulate) {
    for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < n4;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float4 s = accumulate ? out[idx] : make_float4(0.f, 0.f, 0.f, 0.f);
        for (int k = 0; k < S; ++k) {
            const float4 v = __ldg(&part[static_cast<int64_t>(k) * n4 + idx]);
            s.x += v.x;
            s.y += v.y;
            s.z += v.z;
            s.w += v.w;
        }
        out[idx] = s;
    }
}

// ------------------------------------------------------------------ fp32 contraction
constexpr int kFT = 64;   // output tile edge
constexpr int kFTk = 16;  // tokens per step

__global__ void __launch_bounds__(256) gw_f32_kernel(const float* __restrict__ g,
                                                     const float* __restrict__ x, float* GW,
                                                     int64_t N, int d_in, int d_out,
                                                     int accumulate) {
    __shared__ float gs[kFTk][kFT];
    __shared__ float xs[kFTk][kFT];
    const int o0 = blockIdx.y * kFT, k0 = blockIdx.x * kFT;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    float acc[4][4] = {};
    for (int64_t t0 = 0; t0 < N; t0 += kFTk) {
        for (int idx = threadIdx.x; idx < kFTk * kFT; idx += 256) {
            const int tt = idx / kFT, c = idx % kFT;
            const int64_t t = t0 + tt;
            gs[tt][c] = (t < N && o0 + c < d_out) ? g[t * d_out + o0 + c] : 0.f;
            xs[tt][c] = (t < N && k0 + c < d_in) ? x[t * d_in + k0 + c] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int tt = 0; tt < kFTk; ++tt) {
            float gv[4], xv[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                gv[a] = gs[tt][ty * 4 + a];
                xv[a] = xs[tt][tx * 4 + a];
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[a][c] = fmaf(gv[a], xv[c], acc[a][c]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int o = o0 + ty * 4 + a;
        if (o >= d_out) continue;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int k = k0 + tx * 4 + c;
            if (k >= d_in) continue;
            float* dstp = GW + static_cast<int64_t>(o) * d_in + k;
            *dstp = accumulate ? *dstp + acc[a][c] : acc[a][c];
        }
    }
}

int choose_splits(int64_t N, int32_t d_in, int32_t d_out) {
    const int64_t tiles = static_cast<int64_t>((d_out + kGM - 1) / kGM) * ((d_in + kGN - 1) / kGN);
    const int64_t nkb = (N + kGK - 1) / kGK;
    int64_t S = num_sms() / tiles;
    S = std::min<int64_t>(S, nkb / 8);
    return static_cast<int>(std::max<int64_t>(S, 1));
}

}  // namespace

size_t wgrad_workspace_bytes(dust_dtype dt, int64_t N, int32_t d_in, int32_t d_out) {
    if (dt == DUST_BF16) {
        const int S = choose_splits(N, d_in, d_out);
        return align_up(static_cast<size_t>(N) * d_out * 2, 256) +
               (S > 1 ? align_up(static_cast<size_t>(S) * d_out * d_in * 4, 256) : 0);
    }
    return align_up(static_cast<size_t>(N) * d_out * 4, 256);
}

dust_status wgrad_launch(const float* r, int64_t ld_r, const void* x, dust_dtype dt, int64_t N,
                         int32_t d_in, int32_t d_out, int32_t K_chunk, int32_t K_total,
                         float sigma, NoiseKey key, float* G_W, int accumulate, float* g_out,
                         void* ws, cudaStream_t s) {
    const int nq = d_out / 4;
    GhatParams gp;
    gp.r = r;
    gp.ld_r = ld_r;
    gp.N = N;
    gp.d_out = d_out;
    gp.K = K_chunk;
    gp.nqb = (nq + kGThreads - 1) / kGThreads;
    gp.units = N * gp.nqb;
    gp.scale = -1.0f / (static_cast<float>(K_total) * sigma);
    gp.key = key;
    const int64_t max_blocks = static_cast<int64_t>(num_sms()) * 16;
    const unsigned gblocks = static_cast<unsigned>(std::min<int64_t>(gp.units, max_blocks));

    if (dt == DUST_BF16) {
        gp.gb = static_cast<__nv_bfloat16*>(ws);
        gp.gf = g_out;
        prof_begin(s);
        ghat_kernel<<<gblocks, kGThreads, 0, s>>>(gp);
        prof_end(s, "ghat_reduce_draws");
        const int S = choose_splits(N, d_in, d_out);
        CUtensorMap tmg, tmx;
        if (!make_tmap_bf16_2d(&tmg, gp.gb, static_cast<uint64_t>(N), d_out, kGK, 64) ||
            !make_tmap_bf16_2d(&tmx, x, static_cast<uint64_t>(N), d_in, kGK, 64))
            return DUST_ERR_CUDA;
        GwParams p;
        p.ew = device_error_word();
        p.N = N;
        p.d_in = d_in;
        p.d_out = d_out;
        const int64_t nkb = (N + kGK - 1) / kGK;
        p.tokens_per_split = ((nkb + S - 1) / S) * kGK;
        if (S == 1) {
            p.out = G_W;
            p.accumulate = accumulate;
        } else {
            p.out = reinterpret_cast<float*>(static_cast<char*>(ws) +
                                             align_up(static_cast<size_t>(N) * d_out * 2, 256));
            p.accumulate = 0;
        }
        static bool attr_done[64] = {};
        int dev = 0;
        cudaGetDevice(&dev);
        if (dev < 64 && !attr_done[dev]) {
            if (cudaFuncSetAttribute(gw_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kGSmem) != cudaSuccess)
                return DUST_ERR_CUDA;
            attr_done[dev] = true;
        }
        dim3 grid((d_out + kGM - 1) / kGM, (d_in + kGN - 1) / kGN, S);
        prof_begin(s);
        gw_bf16_kernel<<<grid, kGWThreads, kGSmem, s>>>(tmg, tmx, p);
        prof_end(s, "gw_bf16_tcgen05");
        if (S > 1) {
            const int64_t n4 = static_cast<int64_t>(d_out) * d_in / 4;
            const unsigned rb = static_cast<unsigned>(std::min<int64_t>((n4 + 255) / 256, max_blocks));
            prof_begin(s);
            splitk_reduce_kernel<<<rb, 256, 0, s>>>(reinterpret_cast<const float4*>(p.out), S, n4,
                                                    reinterpret_cast<float4*>(G_W), accumulate);
            prof_end(s, "gw_splitk_reduce");
        }
        return cudaGetLastError() == cudaSuccess ? DUST_OK : DUST_ERR_CUDA;
    }
    // fp32: g in fp32 (into g_out when given, else the workspace), SIMT contraction.
    float* gf = g_out ? g_out : static_cast<float*>(ws);
    gp.gb = nullptr;
    gp.gf = gf;
    prof_begin(s);
    ghat_kernel<<<gblocks, kGThreads, 0, s>>>(gp);
    prof_end(s, "ghat_reduce_draws");
    dim3 grid((d_in + kFT - 1) / kFT, (d_out + kFT - 1) / kFT);
    prof_begin(s);
    gw_f32_kernel<<<grid, 256, 0, s>>>(gf, static_cast<const float*>(x), G_W, N, d_in, d_out,
                                       accumulate);
    prof_end(s, "gw_f32_simt");
    return cudaGetLastError() == cudaSuccess ? DUST_OK : DUST_ERR_CUDA;
}

}  // namespace dust
