// Noisy linear forward with the per-draw loss change (Dust review page, section "신용 할당",
// noise equation y_t -> y_t + sigma a_t, with the quadratic readout l = 1/2 |y + sigma a - u|^2).
//
// bf16 layers: one tcgen05 kernel; each CTA owns a 128-token x kBN-channel tile of one layer
// (a launch may hold the tiles of up to kMaxGroup layers, described by a table in parameter
// space; kBN = 256, 192 or 128, chosen per launch so that the tiles fill the last wave of CTAs
// best).  TMA brings x and W tiles (128-byte swizzle, 2-stage ring) into shared memory, one
// thread issues tcgen05.mma into a 128 x kBN fp32 accumulator in tensor memory.  The epilogue
// turns the accumulator into s_e = kKappa sigma (y - u) in place; then the CTA's sixteen warps
// (four groups of four, one warp per TMEM lane quarter in each group) share (draw,
// channel-half) work units: each thread owns one token, regenerates the normals of the unit's
// channels (never stored) and sums sigma a e + sigma^2 a^2 / 2 into a per-unit partial.
// Tiles of the last, partial wave of CTAs are split into unit ranges (each computing the
// tile's GEMM) so that the wave ends together.  The CTA that completes a token block (a
// counter of finished units) adds the partials of all units in a fixed order, so the result
// is deterministic.
//
// fp32 layers: a SIMT kernel (one warp per token, one quad of channels per lane) and a
// partial-sum reduction kernel.
#include <algorithm>
#include <vector>

#include "dust_device.cuh"
#include "dust_internal.h"

namespace dust {
namespace {

constexpr int kBM = 128;  // tokens per tile
constexpr int kBK = 64;   // d_in per pipeline stage (128 bytes of bf16: one swizzle row)
constexpr int kStages = 2;
constexpr int kThreads = 512;  // 4 groups of 4 warps
constexpr int kGroups = kThreads / 128;
constexpr uint32_t kABytes = kBM * kBK * 2;
constexpr uint32_t kTmemCols = 256;
constexpr int kBN = 256;  // channels per tile (the MMA's N)
constexpr uint32_t kStageBytes = kABytes + kBN * kBK * 2;
constexpr uint32_t kSmemBytes = kStages * kStageBytes + 1024 + 256;
constexpr int kMaxGroup = 64;  // layers per grouped launch (parameter space holds their table)

struct FwdLayer {
    const __nv_bfloat16* u;
    float* partial;  // [2 n_tiles, K, N]: (channel tile, half) x draw x token
    float* dloss;    // [K, ld]
    int* counters;   // [m_tiles], zero on entry
    int64_t ld;
    int d_in, d_out, n_tiles, tile_begin;
    uint32_t layer_id;
};

template <int kMax>
struct FwdTable {
    CUtensorMap tmx[kMax];
    CUtensorMap tmw[kMax];
    FwdLayer layer[kMax];
    ErrorWord* ew;
    int64_t N;
    int64_t total_tiles;
    int64_t n_full;  // tiles processed whole, one CTA each (CTAs 0 .. n_full-1)
    int split;       // unit ranges per tile of the remaining tiles
    int n_layers, m_tiles, K;
    float sigma_k;  // kKappa sigma: scales the residual so the noise radius needs no kKappa
    float h_lg2;    // sigma^2 ln 2: the quadratic term per unit of -log2 u
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

template <int kMax>
__global__ void __launch_bounds__(kThreads, 2) fwd_bf16_kernel(const __grid_constant__ FwdTable<kMax> T) {
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
    const int64_t N = T.N;
    const int K = T.K;
    const int U = 2 * K;  // work units per tile: (draw, channel half)

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
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

    // This CTA's tile and unit range: the tiles of the full waves take one CTA each (all
    // units); the tiles of the last, partial wave are split into T.split unit ranges, each
    // computing the tile's GEMM, so that the last wave ends nearly together.
    int tile, u_begin, u_end;
    if (static_cast<int64_t>(blockIdx.x) < T.n_full) {
        tile = blockIdx.x;
        u_begin = 0;
        u_end = U;
    } else {
        const int r = blockIdx.x - static_cast<int>(T.n_full);
        const int part = r % T.split;
        tile = static_cast<int>(T.n_full) + r / T.split;
        u_begin = U * part / T.split;
        u_end = U * (part + 1) / T.split;
    }
    uint32_t kc_prod = 0, kc_mma = 0;
    const uint32_t acc_phase = 0;
    int l = 0;
    {
        while (l + 1 < T.n_layers && tile >= T.layer[l + 1].tile_begin) ++l;
        const FwdLayer& L = T.layer[l];
        const CUtensorMap* tmx = &T.tmx[l];
        const CUtensorMap* tmw = &T.tmw[l];
        const int local = tile - L.tile_begin;
        const int m_tile = local % T.m_tiles;
        const int n_tile = local / T.m_tiles;
        const int64_t m0 = static_cast<int64_t>(m_tile) * kBM;
        const int n0 = n_tile * kBN;
        const int nk = (L.d_in + kBK - 1) / kBK;

        if (warp == 0 && lane == 0) {
            // TMA producer
            prefetch_tensormap(tmx);
            prefetch_tensormap(tmw);
            for (int kb = 0; kb < nk; ++kb, ++kc_prod) {
                const int s = kc_prod % kStages;
                if (kc_prod >= kStages &&
                    !mbar_wait_bounded(&empty[s], ((kc_prod / kStages) - 1) & 1, T.ew, 101))
                    break;
                uint8_t* a = smem + s * kStageBytes;
                mbar_arrive_expect_tx(&full[s], kStageBytes);
                tma_load_2d(a, tmx, &full[s], kb * kBK, static_cast<int32_t>(m0));
                tma_load_2d(a + kABytes, tmw, &full[s], kb * kBK, n0);
            }
        } else if (warp == 1 && lane == 0) {
            // MMA issuer: 4 MMAs of K = 16 per stage; operands K-major, 128-byte swizzle,
            // 8-row core groups 1024 bytes apart.
            constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, 0, 0);
            for (int kb = 0; kb < nk; ++kb, ++kc_mma) {
                const int s = kc_mma % kStages;
                if (!mbar_wait_bounded(&full[s], (kc_mma / kStages) & 1, T.ew, 102)) break;
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

        mbar_wait_bounded(acc_full, acc_phase, T.ew, 103);
        __syncwarp();
        tc_fence_after();

        // ---------------- epilogue: every warp; TMEM lane quarter = warp % 4, and the kGroups
        // warps that share a lane quarter split the work (chunks in phase 1, units in phase 2).
        const int lq = warp & 3;
        const int grp = warp >> 2;
        const int row = lq * 32 + lane;
        const int64_t t = m0 + row;
        const bool valid = t < N;
        const uint32_t trow = tmem + (static_cast<uint32_t>(lq * 32) << 16);
        const int nchunks = min(kBN, L.d_out - n0) / 16;

        // Phase 1: s_e = kKappa sigma (y - u), written back in place.
        for (int c = grp; c < nchunks; c += kGroups) {
            float v[16];
            tmem_ld16(trow + c * 16, v);
            tmem_wait_ld();
            if (valid) {
                const uint4* up =
                    reinterpret_cast<const uint4*>(L.u + t * L.d_out + n0 + c * 16);
                float uf[16];
                unpack_bf16x8(__ldg(up), uf);
                unpack_bf16x8(__ldg(up + 1), uf + 8);
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = T.sigma_k * (v[j] - uf[j]);
            } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = 0.f;
            }
            // stored per channel quad as (e0, e2, e1, e3): phase 2 then loads the pairs
            // (e0, e2) and (e1, e3) that go with the cosines and the sines of the quad's two
            // polar pairs
            float w[16];
#pragma unroll
            for (int j = 0; j < 16; j += 4) {
                w[j] = v[j];
                w[j + 1] = v[j + 2];
                w[j + 2] = v[j + 1];
                w[j + 3] = v[j + 3];
            }
            tmem_st16(trow + c * 16, w);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // Phase 2: this CTA's units of the tile, dealt round-robin to the warp groups.  A unit
        // is (draw, half of the tile's channels): regenerate the noise and sum the loss change
        // over the half's channels.  In polar form a pair (z, z') = kKappa nq (cos, sin)
        // contributes sigma (z e + z' e') + sigma^2 / 2 (z^2 + z'^2)
        //   = nq (cos s_e + sin s_e') - h L,   h = sigma^2 ln 2,  L = log2 u = -nq^2;
        // the quad's two pairs are the two lanes of packed f32x2 operations.
        const uint32_t tg = T.key.token_offset + static_cast<uint32_t>(t);
        const uint32_t qbase = static_cast<uint32_t>(n0 >> 2) + T.key.quad_offset;
        const F2 mh{-T.h_lg2, -T.h_lg2};
        const int half_chunks = (nchunks + 1) / 2;
        for (int unit = u_begin + grp; unit < u_end; unit += kGroups) {
            const int i = unit >> 1;
            const int hf = unit & 1;
            const uint32_t di = T.key.draw_offset + static_cast<uint32_t>(i);
            const PhiloxRun run = philox_run_over_word0(tg, di, L.layer_id, T.key);
            F2 acc[2] = {{0.f, 0.f}, {0.f, 0.f}};
            const int c_end = hf ? nchunks : half_chunks;
            // s_e of a 16-channel chunk in one tensor-memory read, one wait per four quads (two
            // 8-column reads were 1.6% slower on the block stack; the quads alternate between
            // the two accumulators as before, so the sums are the same)
            for (int c = hf ? half_chunks : 0; c < c_end; ++c) {
                float se[16];
                tmem_ld16(trow + c * 16, se);
                tmem_wait_ld();
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const PolarPairs z = box_muller_pairs(philox_word0(qbase + c * 4 + qq, run, T.key));
                    const F2 lc = fma2(z.s, F2{se[4 * qq + 2], se[4 * qq + 3]},
                                       mul2(z.c, F2{se[4 * qq + 0], se[4 * qq + 1]}));
                    acc[qq & 1] = fma2(z.nq, lc, acc[qq & 1]);
                    acc[qq & 1] = fma2(mh, z.L, acc[qq & 1]);
                }
            }
            if (valid)
                L.partial[((static_cast<int64_t>(n_tile) * 2 + hf) * K + i) * N + t] =
                    (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y);
        }

        // Done with the accumulator.  Count the finished units of the token block; the CTA
        // that completes it adds the partials of every unit in a fixed order.
        tc_fence_before();
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) {
            const int done = u_end - u_begin;
            const int old = atomicAdd(&L.counters[m_tile], done);
            *is_last = (old + done == L.n_tiles * U);
        }
        __syncthreads();
        if (*is_last) {
            __threadfence();
            for (int idx = threadIdx.x; idx < K * kBM; idx += kThreads) {
                const int i = idx / kBM;
                const int64_t tt = m0 + (idx % kBM);
                if (tt < N) {
                    float s = 0.f;
                    for (int pp = 0; pp < 2 * L.n_tiles; ++pp)
                        s += __ldcg(&L.partial[(static_cast<int64_t>(pp) * K + i) * N + tt]);
                    L.dloss[static_cast<int64_t>(i) * L.ld + tt] = s;
                }
            }
            if (threadIdx.x == 0) L.counters[m_tile] = 0;
        }
    }

    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

size_t bf16_layer_ws(int64_t N, int32_t d_out, int32_t K) {
    const int64_t n_tiles = (d_out + kBN - 1) / kBN;
    const int64_t m_tiles = (N + kBM - 1) / kBM;
    return align_up(static_cast<size_t>(2 * n_tiles * K * N) * 4, 256) +
           align_up(static_cast<size_t>(m_tiles) * 4, 256);
}

// The form of a launch.  With fewer tiles than three waves of the one-tile kernel (two CTAs
// per SM), the persistent kernel below wins: its GEMM and s_e pass hide behind the noise work
// and its ranges end together (+2% at 8k tokens x 768->3072 in the bench, +43% at 1k tokens).
// With more, the one-tile kernel's 32 noise warps per SM beat the persistent kernel's 28
// (-3% at 32k x 1024^2, -7% for the 48-layer group) and its waves desynchronise by themselves.
// The one-tile kernel cuts each tile of its last, partial wave into `split` unit ranges: a
// range of u units takes ceil(u / kGroups) rounds of its warp groups, and the cost minimised is
// (CTA waves of the tail) x (rounds per range as a share of a whole tile's + the GEMM share of
// a tile, about 6%).
constexpr int kPersistentMaxWaves = 3;

struct FwdPlan {
    bool persistent;
    int split;
};

FwdPlan plan_forward(const FwdLayerArgs* layers, int n, int64_t N, int K, int64_t sms) {
    const int64_t m_tiles = (N + kBM - 1) / kBM;
    int64_t tiles = 0;
    for (int l = 0; l < n; ++l) tiles += m_tiles * ((layers[l].d_out + kBN - 1) / kBN);
    const int64_t slots = 2 * sms;
    if (tiles < kPersistentMaxWaves * slots) return FwdPlan{true, 0};
    const int units = 2 * K;
    const int64_t rem = tiles % slots;
    if (rem == 0) return FwdPlan{false, 1};
    int best = 1;
    double best_t = 1e300;
    const double full_rounds = static_cast<double>((units + kGroups - 1) / kGroups);
    for (int f = 1; f <= 8 && units / f >= 2; ++f) {
        const double waves = static_cast<double>((rem * f + slots - 1) / slots);
        const int max_units = (units + f - 1) / f;
        const double rounds = static_cast<double>((max_units + kGroups - 1) / kGroups);
        const double t = waves * (rounds / full_rounds + 0.06);
        if (t < best_t - 1e-9) {
            best_t = t;
            best = f;
        }
    }
    return FwdPlan{false, best};
}

// Fills and launches one table of up to kMax layers, one tile per CTA.
template <int kMax>
dust_status launch_bf16_table(const FwdLayerArgs* layers, int n, int64_t N, int K, float sigma,
                              const NoiseKey& key, int split, char* ws, cudaStream_t s) {
    FwdTable<kMax> T;  // copied into the launch's parameter space
    T.ew = device_error_word();
    T.N = N;
    T.n_layers = n;
    T.m_tiles = static_cast<int>((N + kBM - 1) / kBM);
    T.K = K;
    T.sigma_k = kKappa * sigma;
    T.h_lg2 = static_cast<float>(0.69314718055994531 * sigma * sigma);
    T.key = key;
    int64_t tiles = 0;
    // the layers' unit counters side by side at the start of the workspace (one memset clears
    // them all), then the layers' partials; the same total as the sum of bf16_layer_ws
    const size_t counters_bytes = align_up(static_cast<size_t>(T.m_tiles) * 4, 256);
    size_t off = static_cast<size_t>(n) * counters_bytes;
    if (cudaMemsetAsync(ws, 0, off, s) != cudaSuccess) return DUST_ERR_CUDA;
    for (int l = 0; l < n; ++l) {
        const FwdLayerArgs& a = layers[l];
        if (!make_tmap_bf16_2d(&T.tmx[l], a.x, static_cast<uint64_t>(N), a.d_in, kBM, kBK) ||
            !make_tmap_bf16_2d(&T.tmw[l], a.W, static_cast<uint64_t>(a.d_out), a.d_in, kBN, kBK))
            return DUST_ERR_CUDA;
        FwdLayer& L = T.layer[l];
        const int n_tiles = (a.d_out + kBN - 1) / kBN;
        L.u = static_cast<const __nv_bfloat16*>(a.u);
        L.partial = reinterpret_cast<float*>(ws + off);
        L.counters = reinterpret_cast<int*>(ws + static_cast<size_t>(l) * counters_bytes);
        L.dloss = a.dloss;
        L.ld = a.ld;
        L.d_in = a.d_in;
        L.d_out = a.d_out;
        L.n_tiles = n_tiles;
        L.tile_begin = static_cast<int>(tiles);
        L.layer_id = a.layer_id;
        tiles += static_cast<int64_t>(n_tiles) * T.m_tiles;
        if (tiles > 2147483647LL) return DUST_ERR_UNSUPPORTED;
        off += align_up(static_cast<size_t>(2 * n_tiles) * K * N * 4, 256);
    }
    static PerContextOnce attr;
    if (!attr.run([] {
            return cudaFuncSetAttribute(fwd_bf16_kernel<kMax>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        kSmemBytes) == cudaSuccess;
        }))
        return DUST_ERR_CUDA;
    // Full waves of two CTAs per SM take whole tiles; the remainder is split (see the kernel).
    T.total_tiles = tiles;
    const int64_t slots = 2LL * num_sms();
    T.n_full = tiles / slots * slots;
    T.split = split;
    const int64_t grid = T.n_full + (tiles - T.n_full) * T.split;
    if (grid > 2147483647LL) return DUST_ERR_UNSUPPORTED;
    prof_begin(s);
    fwd_bf16_kernel<kMax><<<static_cast<unsigned>(grid), kThreads, kSmemBytes, s>>>(T);
    prof_end(s, kMax == 1 ? "fwd_bf16_noise_loss" : "fwd_bf16_noise_loss_grouped");
    return cudaGetLastError() == cudaSuccess ? DUST_OK : DUST_ERR_CUDA;
}

template <int kMax>
dust_status launch_persistent(const FwdLayerArgs* layers, int n, int64_t N, int K, float sigma,
                              const NoiseKey& key, char* ws, cudaStream_t s);

template <int kMax>
dust_status launch_bf16(const FwdLayerArgs* layers, int n, int64_t N, int K, float sigma,
                        const NoiseKey& key, char* ws, cudaStream_t s) {
    const FwdPlan plan = plan_forward(layers, n, N, K, num_sms());
    if (plan.persistent) return launch_persistent<kMax>(layers, n, N, K, sigma, key, ws, s);
    return launch_bf16_table<kMax>(layers, n, N, K, sigma, key, plan.split, ws, s);
}

// ------------------------------------------------------------------------ persistent form
// One CTA per SM walks a balanced, contiguous range of the launch's (tile, unit) items, tiles of
// 128 tokens x 256 channels in token-block-major order.  Two 256-column accumulators let the
// next tile's GEMM and s_e pass run while the noise warps work on the current tile:
//   warps 0-3   the control group: warp 0 lane 0 feeds a 4-stage TMA ring, warp 1 lane 0 issues
//               the MMAs into accumulator jj % 2, then all four warps (one per TMEM lane
//               quarter) rewrite it in place to s_e and signal se_ready; the accumulator of
//               tile jj is reused for tile jj + 2 once the noise warps signal acc_empty;
//   warps 4-31  seven groups of four noise warps: group g takes the CTA's units g, g + 7, ...
//               (draw, channel half), each as in the one-tile kernel above.
// The per-unit partials are added by fwd_reduce_kernel afterwards, in a fixed order.
constexpr int kPThreads = 1024;
constexpr int kPNoiseGroups = (kPThreads - 128) / 128;  // 7
constexpr int kPStages = 4;
constexpr uint32_t kPStageBytes = kStageBytes;
constexpr uint32_t kPSmemBytes = kPStages * kPStageBytes + 1024 + 256;

template <int kMax>
__global__ void __launch_bounds__(kPThreads, 1) fwd_persistent_kernel(const __grid_constant__ FwdTable<kMax> T) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kPStages * kPStageBytes);
    uint64_t* empty = full + kPStages;
    uint64_t* acc_full = empty + kPStages;  // [2]
    uint64_t* se_ready = acc_full + 2;      // [2]
    uint64_t* acc_empty = se_ready + 2;     // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t N = T.N;
    const int K = T.K;
    const int U = 2 * K;

    if (threadIdx.x == 0) {
        for (int st = 0; st < kPStages; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&se_ready[b], 128);
            mbar_init(&acc_empty[b], kPNoiseGroups * 4);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 2 * kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // waits give up together: the first that times out sets the flag, later ones return at once
    auto wait = [&](uint64_t* bar, uint32_t parity, int site) -> bool {
        if (*abort_flag) return false;
        if (mbar_wait_bounded(bar, parity, T.ew, site)) return true;
        *abort_flag = 1;
        return false;
    };
    // the control group's long waits (for the noise warps, and for the GEMM) poll every 256 ns
    auto wait_idle = [&](uint64_t* bar, uint32_t parity, int site) -> bool {
        if (*abort_flag) return false;
        if (mbar_wait_bounded_sleep(bar, parity, T.ew, site, 256)) return true;
        *abort_flag = 1;
        return false;
    };

    // this CTA's items: [ub, ue) of the launch's total_tiles * U (tile-major)
    const int64_t total = T.total_tiles * U;
    const int64_t ub = total * blockIdx.x / gridDim.x;
    const int64_t ue = total * (blockIdx.x + 1) / gridDim.x;
    if (ub < ue) {
        const int64_t tile_first = ub / U;
        const int nt = static_cast<int>((ue - 1) / U - tile_first + 1);
        int l = 0;
        if (warp < 4) {
            // ------------------------------------------------------------ control group
            uint32_t kc_prod = 0, kc_mma = 0;
            const int row = warp * 32 + lane;
            const uint32_t trow0 = tmem + (static_cast<uint32_t>(warp * 32) << 16);
            for (int jj = 0; jj < nt; ++jj) {
                const int64_t gt = tile_first + jj;
                while (l + 1 < T.n_layers && gt >= T.layer[l + 1].tile_begin) ++l;
                const FwdLayer& L = T.layer[l];
                const int local = static_cast<int>(gt - L.tile_begin);
                const int m_tile = local / L.n_tiles;
                const int n_tile = local - m_tile * L.n_tiles;
                const int64_t m0 = static_cast<int64_t>(m_tile) * kBM;
                const int n0 = n_tile * kBN;
                const int nk = (L.d_in + kBK - 1) / kBK;
                const int b = jj & 1;
                if (jj >= 2) {
                    wait_idle(&acc_empty[b], ((jj >> 1) - 1) & 1, 111);
                    tc_fence_after();
                }
                if (warp == 0 && lane == 0) {
                    const CUtensorMap* tmx = &T.tmx[l];
                    const CUtensorMap* tmw = &T.tmw[l];
                    for (int kb = 0; kb < nk; ++kb, ++kc_prod) {
                        const int st = kc_prod % kPStages;
                        if (kc_prod >= kPStages && !wait(&empty[st], ((kc_prod / kPStages) - 1) & 1, 112))
                            break;
                        uint8_t* a = smem + st * kPStageBytes;
                        mbar_arrive_expect_tx(&full[st], kPStageBytes);
                        tma_load_2d(a, tmx, &full[st], kb * kBK, static_cast<int32_t>(m0));
                        tma_load_2d(a + kABytes, tmw, &full[st], kb * kBK, n0);
                    }
                } else if (warp == 1 && lane == 0) {
                    constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, 0, 0);
                    const uint32_t acc = tmem + static_cast<uint32_t>(b * kTmemCols);
                    for (int kb = 0; kb < nk; ++kb, ++kc_mma) {
                        const int st = kc_mma % kPStages;
                        if (!wait(&full[st], (kc_mma / kPStages) & 1, 113)) break;
                        tc_fence_after();
                        const uint32_t a_addr = smem_u32(smem + st * kPStageBytes);
                        const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
                        for (int kk = 0; kk < kBK / 16; ++kk) {
                            const uint64_t ad = sdesc_sw128(a_addr + kk * 32, 16, 1024);
                            const uint64_t bd = sdesc_sw128(b_addr + kk * 32, 16, 1024);
                            umma_bf16(acc, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
                        }
                        umma_commit(&empty[st]);
                    }
                    umma_commit(&acc_full[b]);
                }
                // s_e = kKappa sigma (y - u) in place, each channel quad as (e0, e2, e1, e3);
                // u is read one chunk ahead
                if (warp == 1 && lane == 0)
                    wait(&acc_full[b], (jj >> 1) & 1, 114);
                else
                    wait_idle(&acc_full[b], (jj >> 1) & 1, 114);
                __syncwarp();
                tc_fence_after();
                const int64_t t = m0 + row;
                const bool valid = t < N;
                const uint32_t trow = trow0 + static_cast<uint32_t>(b * kTmemCols);
                const int nchunks = min(kBN, L.d_out - n0) / 16;
                const uint4* up = reinterpret_cast<const uint4*>(L.u + (valid ? t * L.d_out + n0 : 0));
                uint4 un0 = make_uint4(0u, 0u, 0u, 0u), un1 = un0;
                if (valid) {
                    un0 = __ldg(up);
                    un1 = __ldg(up + 1);
                }
                for (int c = 0; c < nchunks; ++c) {
                    float v[16];
                    tmem_ld16(trow + c * 16, v);
                    const uint4 uc0 = un0, uc1 = un1;
                    if (valid && c + 1 < nchunks) {
                        un0 = __ldg(up + 2 * (c + 1));
                        un1 = __ldg(up + 2 * (c + 1) + 1);
                    }
                    tmem_wait_ld();
                    float uf[16];
                    unpack_bf16x8(uc0, uf);
                    unpack_bf16x8(uc1, uf + 8);
                    float w[16];
#pragma unroll
                    for (int j = 0; j < 16; j += 4) {
                        w[j] = valid ? T.sigma_k * (v[j] - uf[j]) : 0.f;
                        w[j + 1] = valid ? T.sigma_k * (v[j + 2] - uf[j + 2]) : 0.f;
                        w[j + 2] = valid ? T.sigma_k * (v[j + 1] - uf[j + 1]) : 0.f;
                        w[j + 3] = valid ? T.sigma_k * (v[j + 3] - uf[j + 3]) : 0.f;
                    }
                    tmem_st16(trow + c * 16, w);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&se_ready[b]);
            }
        } else {
            // ------------------------------------------------------------ noise warps
            const int gi = (warp - 4) >> 2;
            const int lq = warp & 3;
            const int row = lq * 32 + lane;
            const uint32_t trow0 = tmem + (static_cast<uint32_t>(lq * 32) << 16);
            const F2 mh{-T.h_lg2, -T.h_lg2};
            for (int jj = 0; jj < nt; ++jj) {
                const int64_t gt = tile_first + jj;
                while (l + 1 < T.n_layers && gt >= T.layer[l + 1].tile_begin) ++l;
                const FwdLayer& L = T.layer[l];
                const int local = static_cast<int>(gt - L.tile_begin);
                const int m_tile = local / L.n_tiles;
                const int n_tile = local - m_tile * L.n_tiles;
                const int64_t t = static_cast<int64_t>(m_tile) * kBM + row;
                const bool valid = t < N;
                const int n0 = n_tile * kBN;
                const int nchunks = min(kBN, L.d_out - n0) / 16;
                const int half_chunks = (nchunks + 1) / 2;
                const int b = jj & 1;
                const uint32_t trow = trow0 + static_cast<uint32_t>(b * kTmemCols);
                const uint32_t tg = T.key.token_offset + static_cast<uint32_t>(t);
                const uint32_t qbase = static_cast<uint32_t>(n0 >> 2) + T.key.quad_offset;
                // this group's units of the tile: u in [max(ub, gt U), min(ue, (gt + 1) U)) with
                // (u - ub) % 7 == gi
                const int64_t lo = max(ub, gt * U), hi = min(ue, (gt + 1) * U);
                const int64_t first = lo + (gi - (lo - ub) % kPNoiseGroups + kPNoiseGroups) % kPNoiseGroups;
                wait(&se_ready[b], (jj >> 1) & 1, 115);
                tc_fence_after();
                for (int64_t u = first; u < hi; u += kPNoiseGroups) {
                    const int unit = static_cast<int>(u - gt * U);
                    const int i = unit >> 1;
                    const int hf = unit & 1;
                    const uint32_t di = T.key.draw_offset + static_cast<uint32_t>(i);
                    const PhiloxRun run = philox_run_over_word0(tg, di, L.layer_id, T.key);
                    F2 acc[2] = {{0.f, 0.f}, {0.f, 0.f}};
                    const int c_end = hf ? nchunks : half_chunks;
                    for (int c = hf ? half_chunks : 0; c < c_end; ++c) {
#pragma unroll
                        for (int piece = 0; piece < 2; ++piece) {
                            float se[8];
                            tmem_ld8(trow + c * 16 + piece * 8, se);
                            tmem_wait_ld8(se);
#pragma unroll
                            for (int qq = 0; qq < 2; ++qq) {
                                const PolarPairs z = box_muller_pairs(
                                    philox_word0(qbase + c * 4 + piece * 2 + qq, run, T.key));
                                const F2 lc = fma2(z.s, F2{se[4 * qq + 2], se[4 * qq + 3]},
                                                   mul2(z.c, F2{se[4 * qq + 0], se[4 * qq + 1]}));
                                acc[qq] = fma2(z.nq, lc, acc[qq]);
                                acc[qq] = fma2(mh, z.L, acc[qq]);
                            }
                        }
                    }
                    if (valid)
                        L.partial[((static_cast<int64_t>(n_tile) * 2 + hf) * K + i) * N + t] =
                            (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[b]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 2 * kTmemCols);
}

// dloss[i][t] = the sum over the 2 n_tiles unit partials of (draw i, token t), in order.
template <int kMax>
__global__ void __launch_bounds__(256) fwd_reduce_kernel(const __grid_constant__ FwdTable<kMax> T) {
    const FwdLayer& L = T.layer[blockIdx.y];
    const int64_t total = static_cast<int64_t>(T.K) * T.N;
    const int parts = 2 * L.n_tiles;
    for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int i = static_cast<int>(idx / T.N);
        const int64_t t = idx - static_cast<int64_t>(i) * T.N;
        const float* p = L.partial + static_cast<int64_t>(i) * T.N + t;
        const int64_t stride = static_cast<int64_t>(T.K) * T.N;
        float s = 0.f;
        for (int pp = 0; pp < parts; ++pp) s += __ldcs(p + pp * stride);
        L.dloss[static_cast<int64_t>(i) * L.ld + t] = s;
    }
}

template <int kMax>
dust_status launch_persistent(const FwdLayerArgs* layers, int n, int64_t N, int K, float sigma,
                              const NoiseKey& key, char* ws, cudaStream_t s) {
    FwdTable<kMax> T;  // copied into the launch's parameter space
    T.ew = device_error_word();
    T.N = N;
    T.n_layers = n;
    T.m_tiles = static_cast<int>((N + kBM - 1) / kBM);
    T.K = K;
    T.sigma_k = kKappa * sigma;
    T.h_lg2 = static_cast<float>(0.69314718055994531 * sigma * sigma);
    T.key = key;
    T.n_full = 0;
    T.split = 1;
    int64_t tiles = 0;
    size_t off = 0;
    for (int l = 0; l < n; ++l) {
        const FwdLayerArgs& a = layers[l];
        if (!make_tmap_bf16_2d(&T.tmx[l], a.x, static_cast<uint64_t>(N), a.d_in, kBM, kBK) ||
            !make_tmap_bf16_2d(&T.tmw[l], a.W, static_cast<uint64_t>(a.d_out), a.d_in, kBN, kBK))
            return DUST_ERR_CUDA;
        FwdLayer& L = T.layer[l];
        const int n_tiles = (a.d_out + kBN - 1) / kBN;
        L.u = static_cast<const __nv_bfloat16*>(a.u);
        L.partial = reinterpret_cast<float*>(ws + off);
        L.counters = nullptr;
        L.dloss = a.dloss;
        L.ld = a.ld;
        L.d_in = a.d_in;
        L.d_out = a.d_out;
        L.n_tiles = n_tiles;
        L.tile_begin = static_cast<int>(tiles);
        L.layer_id = a.layer_id;
        tiles += static_cast<int64_t>(n_tiles) * T.m_tiles;
        if (tiles > 2147483647LL) return DUST_ERR_UNSUPPORTED;
        off += bf16_layer_ws(N, a.d_out, K);
    }
    T.total_tiles = tiles;
    static PerContextOnce attr;
    if (!attr.run([] {
            return cudaFuncSetAttribute(fwd_persistent_kernel<kMax>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        kPSmemBytes) == cudaSuccess;
        }))
        return DUST_ERR_CUDA;
    const int64_t grid = std::min<int64_t>(num_sms(), tiles * 2 * K);
    prof_begin(s);
    fwd_persistent_kernel<kMax><<<static_cast<unsigned>(grid), kPThreads, kPSmemBytes, s>>>(T);
    prof_end(s, kMax == 1 ? "fwd_bf16_noise_loss" : "fwd_bf16_noise_loss_grouped");
    const int64_t outs = static_cast<int64_t>(K) * N;
    prof_begin(s);
    fwd_reduce_kernel<kMax><<<dim3(static_cast<unsigned>(std::min<int64_t>((outs + 255) / 256,
                                                                           num_sms() * 8LL)),
                                   static_cast<unsigned>(n)),
                              256, 0, s>>>(T);
    prof_end(s, kMax == 1 ? "fwd_reduce_partials" : "fwd_reduce_partials_grouped");
    return cudaGetLastError() == cudaSuccess ? DUST_OK : DUST_ERR_CUDA;
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
            const F4 z = normal_quad(static_cast<uint32_t>(q) + p.key.quad_offset, tg,
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
    if (dt == DUST_BF16) return bf16_layer_ws(N, d_out, K);
    const int64_t n_cb = (d_out + 4 * kF32Quads - 1) / (4 * kF32Quads);
    return align_up(static_cast<size_t>(n_cb * K * N) * 4, 256);
}

void fwd_plan(const int32_t* d_out, int n, int64_t N, int32_t K, int64_t sms, int32_t* persistent,
              int32_t* split) {
    std::vector<FwdLayerArgs> a(static_cast<size_t>(n), FwdLayerArgs{});
    for (int l = 0; l < n; ++l) a[l].d_out = d_out[l];
    const FwdPlan p = plan_forward(a.data(), n, N, K, sms);
    *persistent = p.persistent ? 1 : 0;
    *split = p.split;
}

size_t fwd_grouped_workspace_bytes(const FwdLayerArgs* layers, int n, int64_t N, int32_t K) {
    size_t total = 0;
    for (int l = 0; l < n; ++l) total += bf16_layer_ws(N, layers[l].d_out, K);
    return total;
}

dust_status fwd_grouped_launch(const FwdLayerArgs* layers, int n, int64_t N, int32_t K,
                               float sigma, NoiseKey key, void* ws, cudaStream_t s) {
    char* base = static_cast<char*>(ws);
    for (int l0 = 0; l0 < n; l0 += kMaxGroup) {
        const int cnt = std::min(kMaxGroup, n - l0);
        const dust_status st = launch_bf16<kMaxGroup>(layers + l0, cnt, N, K, sigma, key, base, s);
        if (st != DUST_OK) return st;
        base += fwd_grouped_workspace_bytes(layers + l0, cnt, N, K);
    }
    return DUST_OK;
}

dust_status fwd_launch(const void* x, const void* W, const void* u, dust_dtype dt, int64_t N,
                       int32_t d_in, int32_t d_out, int32_t K, float sigma, NoiseKey key,
                       float* dloss, int64_t ld, void* ws, cudaStream_t s) {
    if (dt == DUST_BF16) {
        const int64_t tiles = (N + kBM - 1) / kBM * ((d_out + kBN - 1) / kBN);
        if (tiles > 2147483647LL) return DUST_ERR_UNSUPPORTED;
        FwdLayerArgs a{x, W, u, d_in, d_out, key.layer, dloss, ld};
        return launch_bf16<1>(&a, 1, N, K, sigma, key, static_cast<char*>(ws), s);
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
