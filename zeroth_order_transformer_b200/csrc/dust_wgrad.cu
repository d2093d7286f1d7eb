// Output-error estimate and weight estimate (Dust review page, section "신용 할당":
// g_t = -(1/(K sigma)) sum_i r_t^(i) a_t^(i) and G_W = sum_t g_t x_t^T).
//
// Stage 1 (ghat_kernel): one thread per (token, two channel quads) regenerates the quads'
// normals for every draw and accumulates the reward-weighted sum; g is written as bf16 (the
// tensor core operand) and optionally as fp32.  With two terms the operand is g's bf16
// rounding hi = bf16(g) in rows [0, N) and the rounding of the remainder lo = bf16(g - hi)
// in rows [N, 2N): hi + lo carries about 16 significant bits instead of 8.  A grid-stride
// loop over units of 128 consecutive (token, quad pair) items of a layer keeps every SM busy
// to the end.
// Stage 2 (gw_bf16_kernel): G_W = g^T x on the tensor cores.  Both operands are MN-major
// (tokens are the contraction index and the slow index of g [N, d_out] and x [N, d_in]):
// TMA loads 64-token x 64-element boxes with 128-byte swizzle.  A CTA owns a 256 x 256
// output tile as two halves of 128 rows, each in its own TMEM accumulator; one thread issues
// tcgen05.mma (M = 128 output rows, N = 256 output columns, K = 16 tokens per instruction)
// for both halves against the same x tile, so x is loaded once per stage for 256 rows; with
// two terms each 16-token step also issues the lo rows into the same accumulators.  When the
// outputs have fewer tiles than SMs the token range is split (split-K) and a fixed-order
// reduction adds the partials, so the result is deterministic.  One launch covers up to
// kMaxGroup layers (tables in parameter space).  fp32 layers use a SIMT tiled contraction on
// the fp32 g.
#include <algorithm>
#include <mutex>

#include "dust_device.cuh"
#include "dust_internal.h"

namespace dust {
namespace {

constexpr int kMaxGroup = 64;

// ------------------------------------------------------------------ stage 1: g
constexpr int kGThreads = 128;
// Grid of the draw reduction, in CTAs per SM.  The CTAs walk the units grid-stride, each with
// an equal share; nine of them (56 registers per thread) fit on an SM at once, so a grid of one
// wave of eight per SM can land unevenly, and a grid of several small waves lets the block
// scheduler even out the SMs' loads as CTAs finish.  48 per SM beat one wave of 8 by 11% and 16
// per SM by 3% on the 48-layer stack; a per-warp start stagger made no difference, so the gain
// is the balance, not the warps' relative phase.
constexpr int kGCtasPerSm = 48;

struct GhatLayer {
    const float* r;
    __nv_bfloat16* gb;  // [N, d_out] (hi) or null
    __nv_bfloat16* gl;  // [N, d_out] (lo, two terms) or null
    float* gf;          // [N, d_out] or null
    int64_t ld_r, unit_begin;
    int64_t n_flat;  // N * ceil(d_out / 8): (token, pair of channel quads) items, token-major
    uint64_t np_magic;  // div_magic(ceil(d_out / 8))
    int d_out;
    uint32_t layer_id;
};

template <int kMax>
struct GhatTable {
    GhatLayer layer[kMax];
    int64_t total_units;
    int n_layers, K;
    float scale;  // -1 / (K_total sigma)
    NoiseKey key;
};

// Each thread owns one token and two consecutive channel quads (the second absent at the end
// of a row with an odd number of quads), so the credit of a draw is loaded once for eight
// channels and the two quads' Philox chains interleave.  (Unrolling the draws as well spills
// at 64 registers; two quads at 53 registers beat one quad with four draws unrolled by 3-7%.)
template <int kMax>
__global__ void __launch_bounds__(kGThreads, 8) ghat_kernel(const __grid_constant__ GhatTable<kMax> T) {
    int l = 0;
    for (int64_t u = blockIdx.x; u < T.total_units; u += gridDim.x) {
        while (l + 1 < T.n_layers && u >= T.layer[l + 1].unit_begin) ++l;
        const GhatLayer& L = T.layer[l];
        // a unit is 128 consecutive (token, quad pair) items, so no lane idles when the row's
        // pair count is not a multiple of 128
        const int64_t f = (u - L.unit_begin) * kGThreads + threadIdx.x;
        if (f >= L.n_flat) continue;
        const int nq = L.d_out >> 2;
        const int np = (nq + 1) >> 1;
        const int64_t t = div_by_magic(f, np, L.np_magic);
        const int q = 2 * static_cast<int>(f - t * np);
        const bool two = q + 1 < nq;
        const uint32_t tg = T.key.token_offset + static_cast<uint32_t>(t);
        const uint32_t qg = static_cast<uint32_t>(q) + T.key.quad_offset;
        // per quad, channel pairs (4q, 4q+2) and (4q+1, 4q+3): the lanes of packed f32x2 operations
        F2 a02{0.f, 0.f}, a13{0.f, 0.f}, b02{0.f, 0.f}, b13{0.f, 0.f};
        const float* rt = L.r + t;
        const PhiloxRun run_z = philox_run_over_word2(qg, tg, L.layer_id, T.key);
        const PhiloxRun run_w = philox_run_over_word2(qg + 1, tg, L.layer_id, T.key);
#pragma unroll 1
        for (int i = 0; i < T.K; ++i) {
            const float ri = __ldg(rt + static_cast<int64_t>(i) * L.ld_r);
            const uint32_t di = T.key.draw_offset + static_cast<uint32_t>(i);
            const PolarPairs z = box_muller_pairs(philox_word2(di, run_z, T.key));
            const PolarPairs w = box_muller_pairs(philox_word2(di, run_w, T.key));
            // r a = kKappa (r nq) (cos, sin) per pair; kKappa is applied with the scale
            const F2 rz = mul2(F2{ri, ri}, z.nq);
            const F2 rw = mul2(F2{ri, ri}, w.nq);
            a02 = fma2(rz, z.c, a02);
            a13 = fma2(rz, z.s, a13);
            b02 = fma2(rw, w.c, b02);
            b13 = fma2(rw, w.s, b13);
        }
        const float sk = T.scale * kKappa;
        const float4 ga = make_float4(a02.x * sk, a13.x * sk, a02.y * sk, a13.y * sk);
        const float4 gb = make_float4(b02.x * sk, b13.x * sk, b02.y * sk, b13.y * sk);
        const int64_t off = t * L.d_out + 4 * q;
        if (L.gb) {
            __nv_bfloat162 h[4] = {__floats2bfloat162_rn(ga.x, ga.y), __floats2bfloat162_rn(ga.z, ga.w),
                                   __floats2bfloat162_rn(gb.x, gb.y), __floats2bfloat162_rn(gb.z, gb.w)};
            const uint32_t* hv = reinterpret_cast<const uint32_t*>(h);
            if (two)
                *reinterpret_cast<uint4*>(L.gb + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
            else
                *reinterpret_cast<uint2*>(L.gb + off) = make_uint2(hv[0], hv[1]);
            if (L.gl) {
                // the remainder g - hi is exact in fp32 (|g - hi| <= half a bf16 ulp of g)
                const float2 f0 = __bfloat1622float2(h[0]), f1 = __bfloat1622float2(h[1]);
                const float2 f2 = __bfloat1622float2(h[2]), f3 = __bfloat1622float2(h[3]);
                __nv_bfloat162 lo[4] = {__floats2bfloat162_rn(ga.x - f0.x, ga.y - f0.y),
                                        __floats2bfloat162_rn(ga.z - f1.x, ga.w - f1.y),
                                        __floats2bfloat162_rn(gb.x - f2.x, gb.y - f2.y),
                                        __floats2bfloat162_rn(gb.z - f3.x, gb.w - f3.y)};
                const uint32_t* lv = reinterpret_cast<const uint32_t*>(lo);
                if (two)
                    *reinterpret_cast<uint4*>(L.gl + off) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
                else
                    *reinterpret_cast<uint2*>(L.gl + off) = make_uint2(lv[0], lv[1]);
            }
        }
        if (L.gf) {
            *reinterpret_cast<float4*>(L.gf + off) = ga;
            if (two) *reinterpret_cast<float4*>(L.gf + off + 4) = gb;
        }
    }
}

// ------------------------------------------------------------------ stage 2: G_W (bf16)
constexpr int kGH = 128;  // output rows (o) per MMA (one TMEM accumulator)
constexpr int kGM = 256;  // output rows per tile: two MMA halves that share the x tile
constexpr int kGN = 256;  // output columns (k) per tile
constexpr int kGK = 64;   // token granularity of the split-K ranges (a multiple of every stage)
constexpr int kGWThreads = 128;
constexpr uint32_t kGTmemCols = 512;  // two 128 x 256 fp32 accumulators
// Pipeline shape for one or two g terms.  A stage holds kK tokens of both halves' g tiles of
// every term and of the x tile, in boxes of kK tokens x 64 elements: one term, 64-token stages
// (64 KB, three of them); two terms, 32-token stages (48 KB, four of them), whose longer
// look-ahead made the two-term contraction 3-4% faster while one term, with half the MMAs per
// stage, lost 14% at 32 tokens.
template <int kTerms>
struct GwShape {
    static constexpr int kK = kTerms == 1 ? 64 : 32;
    static constexpr uint32_t kBox = kK * 64 * 2;         // one kK-token x 64-element box
    static constexpr uint32_t kHBytes = kGH / 64 * kBox;  // one half's g tile of one term
    static constexpr uint32_t kBBytes = kGN / 64 * kBox;  // the x tile
    static constexpr uint32_t kStageBytes = kTerms * 2 * kHBytes + kBBytes;
    static constexpr int kStages = kTerms == 1 ? 3 : 4;
    static constexpr uint32_t kSmem = kStages * kStageBytes + 1024 + 256;
};
static_assert(GwShape<1>::kSmem <= 227 * 1024 && GwShape<2>::kSmem <= 227 * 1024,
              "pipeline exceeds shared memory");
static_assert(kGK % GwShape<1>::kK == 0 && kGK % GwShape<2>::kK == 0,
              "split-K ranges must hold whole stages");

struct GwLayer {
    float* out;  // G_W (splits == 1; may be null when an optimizer step consumes it) or
                 // partial [S, d_out, d_in]
    OptTargets opt;  // used when the table's optimizer kind is set and splits == 1
    int64_t tokens_per_split;
    int d_in, d_out, o_tiles, k_tiles, splits, tile_begin, accumulate;
};

template <int kMax>
struct GwTable {
    CUtensorMap tmg[kMax];
    CUtensorMap tmx[kMax];
    GwLayer layer[kMax];
    OptParams opt;  // kind 0: no optimizer step
    ErrorWord* ew;
    int64_t N;
    int n_layers;
};

template <int kMax, int kTerms>
__global__ void __launch_bounds__(kGWThreads, 1) gw_bf16_kernel(const __grid_constant__ GwTable<kMax> T) {
    constexpr int kGStages = GwShape<kTerms>::kStages;
    constexpr uint32_t kGStageBytes = GwShape<kTerms>::kStageBytes;
    constexpr int kK = GwShape<kTerms>::kK;
    constexpr uint32_t kBox = GwShape<kTerms>::kBox;
    constexpr uint32_t kGHBytes = GwShape<kTerms>::kHBytes;
    constexpr uint32_t kGBBytes = GwShape<kTerms>::kBBytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGStages * kGStageBytes);
    uint64_t* empty = full + kGStages;
    uint64_t* acc_full = empty + kGStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);

    int l = 0;
    const int tile = blockIdx.x;
    while (l + 1 < T.n_layers && tile >= T.layer[l + 1].tile_begin) ++l;
    const GwLayer& L = T.layer[l];
    const CUtensorMap* tmg = &T.tmg[l];
    const CUtensorMap* tmx = &T.tmx[l];
    const int local = tile - L.tile_begin;
    const int per_split = L.o_tiles * L.k_tiles;
    const int split = local / per_split;
    const int o0 = (local % per_split % L.o_tiles) * kGM;
    const int k0 = (local % per_split / L.o_tiles) * kGN;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t_begin = static_cast<int64_t>(split) * L.tokens_per_split;
    const int64_t t_end = min(T.N, t_begin + L.tokens_per_split);
    const int nk = t_end > t_begin ? static_cast<int>((t_end - t_begin + kK - 1) / kK) : 0;

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

    // rows o0 .. o0 + 127 (half 0) and o0 + 128 .. o0 + 255 (half 1, skipped when the layer
    // ends before it)
    const int halves = o0 + kGH < L.d_out ? 2 : 1;
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(tmg);
        prefetch_tensormap(tmx);
        const uint32_t bytes = static_cast<uint32_t>(kTerms * halves) * kGHBytes + kGBBytes;
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % kGStages;
            if (kb >= kGStages &&
                !mbar_wait_bounded(&empty[s], ((kb / kGStages) - 1) & 1, T.ew, 201))
                break;
            uint8_t* a = smem + s * kGStageBytes;
            uint8_t* bsm = a + kTerms * 2 * kGHBytes;
            const int32_t tok = static_cast<int32_t>(t_begin + static_cast<int64_t>(kb) * kK);
            mbar_arrive_expect_tx(&full[s], bytes);
            // term tm's half h at a + (tm * 2 + h) * kGHBytes; the lo term's rows start at N
            // (rows past 2N read zeros, and hi rows past N, the lo block, meet x rows past N,
            // which read zeros)
            for (int tm = 0; tm < kTerms; ++tm) {
                const int32_t trow = tm == 0 ? tok : static_cast<int32_t>(T.N) + tok;
                for (int h = 0; h < halves; ++h)
#pragma unroll
                    for (int j = 0; j < kGH / 64; ++j)
                        tma_load_2d(a + (tm * 2 + h) * kGHBytes + j * kBox, tmg, &full[s],
                                    o0 + kGH * h + 64 * j, trow);
            }
#pragma unroll
            for (int j = 0; j < kGN / 64; ++j)
                tma_load_2d(bsm + j * kBox, tmx, &full[s], k0 + 64 * j, tok);
        }
    } else if (warp == 1 && lane == 0) {
        // MN-major operands: 64-element (128-byte) rows, one row per token; 8-token core
        // groups 1024 bytes apart (SBO); successive 64-element column blocks one box apart
        // (LBO); 16 tokens per instruction = 2048 bytes.  Half h accumulates in columns
        // [256 h, 256 h + 256) of the CTA's tensor memory.
        constexpr uint32_t idesc = idesc_bf16_f32(kGH, kGN, 1, 1);
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % kGStages;
            if (!mbar_wait_bounded(&full[s], (kb / kGStages) & 1, T.ew, 202)) break;
            tc_fence_after();
            const uint32_t a_addr = smem_u32(smem + s * kGStageBytes);
            const uint32_t b_addr = a_addr + kTerms * 2 * kGHBytes;
#pragma unroll
            for (int kk = 0; kk < kK / 16; ++kk) {
                const uint64_t bd = sdesc_sw128(b_addr + kk * 2048, kBox, 1024);
                for (int h = 0; h < halves; ++h)
#pragma unroll
                    for (int tm = 0; tm < kTerms; ++tm) {
                        const uint64_t ad = sdesc_sw128(
                            a_addr + (tm * 2 + h) * kGHBytes + kk * 2048, kBox, 1024);
                        umma_bf16(tmem + static_cast<uint32_t>(h * 256), ad, bd, idesc,
                                  (kb | kk | tm) != 0 ? 1u : 0u);
                    }
            }
            umma_commit(&empty[s]);
        }
        umma_commit(acc_full);
    }

    mbar_wait_bounded(acc_full, 0, T.ew, 203);
    __syncwarp();
    tc_fence_after();

    const int ncols = min(kGN, L.d_in - k0);
    float* dst = L.out ? L.out + static_cast<int64_t>(split) * L.d_out * L.d_in : nullptr;
    for (int h = 0; h < halves; ++h) {
        const int o = o0 + kGH * h + warp * 32 + lane;
        const uint32_t trow =
            tmem + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(h * 256);
        for (int c = 0; c < ncols / 16; ++c) {
            float v[16];
            tmem_ld16(trow + c * 16, v);
            tmem_wait_ld();
            if (nk == 0) {
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = 0.f;
            }
            if (o < L.d_out) {
                const int64_t e0 = static_cast<int64_t>(o) * L.d_in + k0 + c * 16;
                float4* d4 = dst ? reinterpret_cast<float4*>(dst + e0) : nullptr;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float4 w = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                    if (L.accumulate) {
                        const float4 old = d4[j];
                        w.x += old.x;
                        w.y += old.y;
                        w.z += old.z;
                        w.w += old.w;
                    }
                    if (d4) d4[j] = w;
                    if (T.opt.kind != 0 && L.splits == 1)
                        opt_update4(T.opt, L.opt, e0 + 4 * j, w);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, kGTmemCols);
}

struct SplitLayer {
    const float4* part;  // [S, n4]
    float4* out;         // [n4], or null when an optimizer step consumes the sum
    OptTargets opt;
    int64_t n4;
    int S, accumulate;
};

template <int kMax>
struct SplitTable {
    SplitLayer layer[kMax];
    OptParams opt;
};

// out = (accumulate ? out : 0) + sum_s part[s] in order s = 0 .. S-1, then the optimizer step
// on that sum when one is set; blockIdx.y = layer.
template <int kMax>
__global__ void splitk_reduce_kernel(const __grid_constant__ SplitTable<kMax> T) {
    const SplitLayer& L = T.layer[blockIdx.y];
    for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < L.n4;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float4 s = L.accumulate ? L.out[idx] : make_float4(0.f, 0.f, 0.f, 0.f);
        for (int k = 0; k < L.S; ++k) {
            const float4 v = __ldg(&L.part[static_cast<int64_t>(k) * L.n4 + idx]);
            s.x += v.x;
            s.y += v.y;
            s.z += v.z;
            s.w += v.w;
        }
        if (L.out) L.out[idx] = s;
        if (T.opt.kind != 0) opt_update4(T.opt, L.opt, 4 * idx, s);
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

int64_t gw_tiles(int32_t d_in, int32_t d_out) {
    return static_cast<int64_t>((d_out + kGM - 1) / kGM) * ((d_in + kGN - 1) / kGN);
}

// Split factor for a launch whose layers have `tiles` output tiles in total: fill the SMs once,
// keeping at least 8 token blocks of 64 per split.
int choose_splits(int64_t tiles, int64_t N) {
    const int64_t nkb = (N + kGK - 1) / kGK;
    int64_t S = num_sms() / std::max<int64_t>(tiles, 1);
    S = std::min<int64_t>(S, nkb / 8);
    return static_cast<int>(std::max<int64_t>(S, 1));
}

// bf16 g operand: always room for two terms (hi rows [0, N), lo rows [N, 2N)), so a workspace
// sized once serves either form.
size_t g_operand_bytes(int64_t N, int32_t d_out) {
    return align_up(static_cast<size_t>(2 * N) * d_out * 2, 256);
}

size_t bf16_layer_ws(int64_t N, int32_t d_in, int32_t d_out, int S) {
    return g_operand_bytes(N, d_out) +
           (S > 1 ? align_up(static_cast<size_t>(S) * d_out * d_in * 4, 256) : 0);
}

template <int kMax, int kTerms>
dust_status launch_gw(const GwTable<kMax>& W, int64_t tiles, cudaStream_t s) {
    static PerContextOnce attr;
    if (!attr.run([] {
            return cudaFuncSetAttribute(gw_bf16_kernel<kMax, kTerms>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        GwShape<kTerms>::kSmem) == cudaSuccess;
        }))
        return DUST_ERR_CUDA;
    gw_bf16_kernel<kMax, kTerms><<<static_cast<unsigned>(tiles), kGWThreads,
                                   GwShape<kTerms>::kSmem, s>>>(W);
    return DUST_OK;
}

template <int kMax>
dust_status launch_bf16_tables(const WgradLayerArgs* layers, int n, int64_t N, int32_t K_chunk,
                               int32_t K_total, float sigma, const NoiseKey& key, int accumulate,
                               int g_terms, char* ws, cudaStream_t s,
                               const OptParams* opt = nullptr,
                               const OptTargets* targets = nullptr) {
    int64_t tiles0 = 0;
    for (int l = 0; l < n; ++l) tiles0 += gw_tiles(layers[l].d_in, layers[l].d_out);
    const int S = choose_splits(tiles0, N);
    const int64_t nkb = (N + kGK - 1) / kGK;
    const int64_t tps = ((nkb + S - 1) / S) * kGK;

    // stage 1: g for every layer
    GhatTable<kMax> G;
    G.n_layers = n;
    G.K = K_chunk;
    G.scale = -1.0f / (static_cast<float>(K_total) * sigma);
    G.key = key;
    int64_t units = 0;
    size_t off = 0;
    for (int l = 0; l < n; ++l) {
        const WgradLayerArgs& a = layers[l];
        GhatLayer& L = G.layer[l];
        L.r = a.r;
        L.ld_r = a.ld_r;
        L.gb = reinterpret_cast<__nv_bfloat16*>(ws + off);
        L.gl = g_terms == 2 ? L.gb + N * a.d_out : nullptr;
        L.gf = a.g_out;
        L.d_out = a.d_out;
        L.n_flat = N * ((a.d_out / 4 + 1) / 2);
        L.np_magic = div_magic((a.d_out / 4 + 1) / 2);
        L.unit_begin = units;
        L.layer_id = a.layer_id;
        units += (L.n_flat + kGThreads - 1) / kGThreads;
        off += bf16_layer_ws(N, a.d_in, a.d_out, S);
    }
    G.total_units = units;
    const int64_t max_blocks = static_cast<int64_t>(num_sms()) * kGCtasPerSm;
    prof_begin(s);
    ghat_kernel<kMax><<<static_cast<unsigned>(std::min(units, max_blocks)), kGThreads, 0, s>>>(G);
    prof_end(s, kMax == 1 ? "ghat_reduce_draws" : "ghat_reduce_draws_grouped");

    // stage 2: G_W for every layer
    GwTable<kMax> W;
    W.opt = opt ? *opt : OptParams{};
    W.ew = device_error_word();
    W.N = N;
    W.n_layers = n;
    SplitTable<kMax> R;
    R.opt = W.opt;
    int n_split_layers = 0;
    int64_t max_n4 = 0;
    int64_t tiles = 0;
    off = 0;
    for (int l = 0; l < n; ++l) {
        const WgradLayerArgs& a = layers[l];
        const uint32_t box = g_terms == 2 ? GwShape<2>::kK : GwShape<1>::kK;
        if (!make_tmap_bf16_2d(&W.tmg[l], ws + off, static_cast<uint64_t>(g_terms * N), a.d_out,
                               box, 64) ||
            !make_tmap_bf16_2d(&W.tmx[l], a.x, static_cast<uint64_t>(N), a.d_in, box, 64))
            return DUST_ERR_CUDA;
        GwLayer& L = W.layer[l];
        L.o_tiles = (a.d_out + kGM - 1) / kGM;
        L.k_tiles = (a.d_in + kGN - 1) / kGN;
        L.splits = S;
        L.tokens_per_split = tps;
        L.d_in = a.d_in;
        L.d_out = a.d_out;
        L.tile_begin = static_cast<int>(tiles);
        L.opt = targets ? targets[l] : OptTargets{};
        tiles += static_cast<int64_t>(L.o_tiles) * L.k_tiles * S;
        if (tiles > 2147483647LL) return DUST_ERR_UNSUPPORTED;
        if (S == 1) {
            L.out = a.G_W;
            L.accumulate = accumulate;
        } else {
            L.out = reinterpret_cast<float*>(ws + off + g_operand_bytes(N, a.d_out));
            L.accumulate = 0;
            SplitLayer& Rl = R.layer[n_split_layers++];
            Rl.part = reinterpret_cast<const float4*>(L.out);
            Rl.out = reinterpret_cast<float4*>(a.G_W);
            Rl.opt = L.opt;
            Rl.n4 = static_cast<int64_t>(a.d_out) * a.d_in / 4;
            Rl.S = S;
            Rl.accumulate = accumulate;
            max_n4 = std::max(max_n4, Rl.n4);
        }
        off += bf16_layer_ws(N, a.d_in, a.d_out, S);
    }
    prof_begin(s);
    const dust_status gst = g_terms == 2 ? launch_gw<kMax, 2>(W, tiles, s)
                                         : launch_gw<kMax, 1>(W, tiles, s);
    prof_end(s, kMax == 1 ? "gw_bf16_tcgen05" : "gw_bf16_tcgen05_grouped");
    if (gst != DUST_OK) return gst;
    if (n_split_layers > 0) {
        const unsigned bx = static_cast<unsigned>(
            std::min<int64_t>((max_n4 + 255) / 256, std::max<int64_t>(1, max_blocks / n_split_layers)));
        prof_begin(s);
        splitk_reduce_kernel<kMax><<<dim3(bx, n_split_layers), 256, 0, s>>>(R);
        prof_end(s, kMax == 1 ? "gw_splitk_reduce" : "gw_splitk_reduce_grouped");
    }
    return cudaGetLastError() == cudaSuccess ? DUST_OK : DUST_ERR_CUDA;
}

}  // namespace

size_t wgrad_workspace_bytes(dust_dtype dt, int64_t N, int32_t d_in, int32_t d_out) {
    if (dt == DUST_BF16) return bf16_layer_ws(N, d_in, d_out, choose_splits(gw_tiles(d_in, d_out), N));
    return align_up(static_cast<size_t>(N) * d_out * 4, 256);
}

size_t wgrad_grouped_workspace_bytes(const WgradLayerArgs* layers, int n, int64_t N) {
    size_t total = 0;
    for (int l0 = 0; l0 < n; l0 += kMaxGroup) {
        const int cnt = std::min(kMaxGroup, n - l0);
        int64_t tiles = 0;
        for (int l = l0; l < l0 + cnt; ++l) tiles += gw_tiles(layers[l].d_in, layers[l].d_out);
        const int S = choose_splits(tiles, N);
        for (int l = l0; l < l0 + cnt; ++l)
            total += bf16_layer_ws(N, layers[l].d_in, layers[l].d_out, S);
    }
    return total;
}

dust_status wgrad_grouped_launch(const WgradLayerArgs* layers, int n, int64_t N, int32_t K_chunk,
                                 int32_t K_total, float sigma, NoiseKey key, int accumulate,
                                 int g_terms, void* ws, cudaStream_t s) {
    char* base = static_cast<char*>(ws);
    for (int l0 = 0; l0 < n; l0 += kMaxGroup) {
        const int cnt = std::min(kMaxGroup, n - l0);
        const dust_status st = launch_bf16_tables<kMaxGroup>(layers + l0, cnt, N, K_chunk, K_total,
                                                             sigma, key, accumulate, g_terms, base,
                                                             s);
        if (st != DUST_OK) return st;
        base += wgrad_grouped_workspace_bytes(layers + l0, cnt, N);
    }
    return DUST_OK;
}

dust_status wgrad_launch(const float* r, int64_t ld_r, const void* x, dust_dtype dt, int64_t N,
                         int32_t d_in, int32_t d_out, int32_t K_chunk, int32_t K_total,
                         float sigma, NoiseKey key, float* G_W, int accumulate, float* g_out,
                         int g_terms, void* ws, cudaStream_t s, const OptParams* opt,
                         const OptTargets* targets) {
    if (dt == DUST_BF16) {
        WgradLayerArgs a{r, ld_r, x, d_in, d_out, key.layer, G_W, g_out};
        return launch_bf16_tables<1>(&a, 1, N, K_chunk, K_total, sigma, key, accumulate, g_terms,
                                     static_cast<char*>(ws), s, opt, targets);
    }
    if (opt) return DUST_ERR_UNSUPPORTED;  // fp32 layers: call dust_optimizer_step
    // fp32: g in fp32 (into g_out when given, else the workspace), SIMT contraction.
    float* gf = g_out ? g_out : static_cast<float*>(ws);
    GhatTable<1> G;
    G.n_layers = 1;
    G.K = K_chunk;
    G.scale = -1.0f / (static_cast<float>(K_total) * sigma);
    G.key = key;
    G.layer[0] = GhatLayer{r, nullptr, nullptr, gf, ld_r, 0, N * ((d_out / 4 + 1) / 2),
                           div_magic((d_out / 4 + 1) / 2), d_out, key.layer};
    G.total_units = (G.layer[0].n_flat + kGThreads - 1) / kGThreads;
    const int64_t max_blocks = static_cast<int64_t>(num_sms()) * kGCtasPerSm;
    prof_begin(s);
    ghat_kernel<1><<<static_cast<unsigned>(std::min(G.total_units, max_blocks)), kGThreads, 0, s>>>(G);
    prof_end(s, "ghat_reduce_draws");
    dim3 grid((d_in + kFT - 1) / kFT, (d_out + kFT - 1) / kFT);
    prof_begin(s);
    gw_f32_kernel<<<grid, 256, 0, s>>>(gf, static_cast<const float*>(x), G_W, N, d_in, d_out,
                                       accumulate);
    prof_end(s, "gw_f32_simt");
    return cudaGetLastError() == cudaSuccess ? DUST_OK : DUST_ERR_CUDA;
}

}  // namespace dust
