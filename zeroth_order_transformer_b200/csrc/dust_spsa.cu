// SPSA / MeZO weight-space probe, the contrast estimator (thakicloud page on zero-order
// training, the SPSA paragraph: two forwards, with a perturbation of all weights added and
// subtracted, estimate the gradient; gist.science 2605.15622 and the FedSPZO page: the
// perturbation is regenerated from a shared seed, so only scalars travel).
//
// Probe j moves the weight matrix along z_j [d_out, d_in], drawn from the noise generator in
// its own counter space, (k >> 2, o, probe, layer | 2^31), and stored at the weights' precision
// (bf16).  For the quadratic readout the two perturbed forwards of a probe share y = W x:
//   L_+- = sum_t 1/2 |e_t +- eps v_t|^2,  e_t = W x_t - u_t,  v_t = z_j x_t,
// so L_+ - L_- = 2 eps sum_t <e_t, v_t> and L_+ + L_- = 2 L_0 + eps^2 sum_t |v_t|^2.  The
// kernels evaluate both forwards through those sums, without the cancellation of subtracting
// two large fp32 losses:
//   spsa_dir_kernel     z_j for all probes, bf16, into the workspace [P, d_out_pad, d_in]
//                       (rows d_out .. d_out_pad - 1 of each probe are zero).
//   spsa_gemm_kernel    tcgen05 GEMM of x against W (residual mode: e = y - u and 1/2 |e|^2),
//                       TMA-fed, accumulator in tensor memory, two CTAs per SM.  Its second
//                       epilogue writes the perturbed outputs y + sigma a of every draw
//                       (dust_noisy_linear_output).
//   spsa_probe_gemm_kernel  the same against the stacked directions (probe mode: <e, v> and
//                       |v|^2 per token and 256-row tile), persistent and warp-specialised with
//                       two accumulators, so each tile's epilogue overlaps the next tile's
//                       mainloop.  Tiles run token-tile fastest, so each direction tile is read
//                       once and one output tile's e stays in L2 across the probes.
//   spsa_reduce_kernel  fixed-order sums over tokens and tiles: p_j = (L_+ - L_-) / (2 eps),
//                       L_+ and L_-.
//   spsa_estimate_kernel  G (+)= (1/P_total) sum_j p_j z_j, regenerating z (ALU-bound).
#include <algorithm>

#include "dust_device.cuh"
#include "dust_internal.h"

namespace dust {
namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 64;
constexpr int kStages = 2;  // two CTAs per SM: one's epilogue overlaps the other's mainloop
constexpr int kThreads = 256;  // two warp groups share the epilogue's 16-column chunks
constexpr uint32_t kABytes = kBM * kBK * 2;
constexpr uint32_t kBBytes = kBN * kBK * 2;
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kSmemBytes = kStages * kStageBytes + 1024 + 256 + kBM * 4;
constexpr uint32_t kEBoxBytes = 32 * kBM * 4;  // one staged 32-column box of e
static_assert(4 * kEBoxBytes <= kStages * kStageBytes, "e staging reuses the pipeline buffers");
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kWeightSpace = 0x80000000u;

int pad256(int d) { return (d + kBN - 1) / kBN * kBN; }

// ---------------------------------------------------------------- directions
// One warp per row (probe j, output channel o) of the stacked directions, its lanes over the
// row's channel quads: 256 contiguous bytes per warp store, and 32-bit index arithmetic (the
// host guarantees P d_out_pad < 2^31).
__global__ void __launch_bounds__(256) spsa_dir_kernel(const __grid_constant__ NoiseKey key, int P,
                                                       int d_out, int d_out_pad, int d_in,
                                                       __nv_bfloat16* Z) {
    const int nq = d_in >> 2;
    const int rows = P * d_out_pad;
    const int lane = threadIdx.x & 31;
    const int wpb = blockDim.x >> 5;
    for (int row = blockIdx.x * wpb + (threadIdx.x >> 5); row < rows; row += gridDim.x * wpb) {
        const int o = row % d_out_pad;
        const uint32_t di = key.draw_offset + static_cast<uint32_t>(row / d_out_pad);
        uint2* zr = reinterpret_cast<uint2*>(Z + static_cast<int64_t>(row) * d_in);
        const PhiloxRun run = philox_run_over_word0(static_cast<uint32_t>(o), di,
                                                    key.layer | kWeightSpace, key);
        for (int q = lane; q < nq; q += 32) {
            uint2 out = make_uint2(0u, 0u);
            if (o < d_out) {
                // z = kKappa nq (cos, sin) per pair; lanes: the quad's two pairs
                const PolarPairs z = box_muller_pairs(philox_word0(static_cast<uint32_t>(q), run, key));
                const F2 r = mul2(F2{kKappa, kKappa}, z.nq);
                const F2 zc = mul2(r, z.c), zs = mul2(r, z.s);  // (z0, z2), (z1, z3)
                __nv_bfloat162 lo = __floats2bfloat162_rn(zc.x, zs.x);
                __nv_bfloat162 hi = __floats2bfloat162_rn(zc.y, zs.y);
                out.x = *reinterpret_cast<uint32_t*>(&lo);
                out.y = *reinterpret_cast<uint32_t*>(&hi);
            }
            zr[q] = out;
        }
    }
}

// ---------------------------------------------------------------- GEMM with two epilogues
struct GemmArgs {
    CUtensorMap tmx;  // x [N, d_in], 64 x 128 boxes
    CUtensorMap tmb;  // W [d_out, d_in] or Z [P d_out_pad, d_in], 64 x 256 boxes
    CUtensorMap tme;  // residual mode: e [N, d_out] fp32, 32 x 128 boxes, 128-byte swizzle
    const __nv_bfloat16* u;
    float* e;         // [N, d_out] fp32: written in residual mode, read in probe mode
    float* part_a;    // residual: [o_tiles, N] 1/2 |e|^2;  probe: [2 P o_tiles, N] <e, v>
    float* part_b;    // probe: [2 P o_tiles, N] |v|^2
    void* y_out;      // noisy-output mode: [K, N, ld_out] of y + sigma a, fp32 or bf16
    ErrorWord* ew;
    int64_t N, ld_out;
    int d_in, d_out, o_tiles, P, m_tiles;
    int K, out_bf16;
    float sigma;
    NoiseKey key;
};

// Epilogues of the one-tile GEMM y = x W^T: kResidual writes e = y - u and 1/2 |e|^2 per
// token and tile; kNoisyOut writes y + sigma a_t^(i) for every draw i (the perturbed layer
// outputs, for callers that evaluate their own loss downstream).
enum GemmMode { kResidual = 0, kNoisyOut = 1 };

template <int kMode>
__global__ void __launch_bounds__(kThreads, 2) spsa_gemm_kernel(const __grid_constant__ GemmArgs A) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
    uint64_t* empty = full + kStages;
    uint64_t* acc_full = empty + kStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
    float* red = reinterpret_cast<float*>(smem + kStages * kStageBytes + 256);  // [kBM]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // tile order: token tile fastest, so a tile of W is read once for all token tiles
    const int m_tile = blockIdx.x % A.m_tiles;
    const int o_tile = blockIdx.x / A.m_tiles;
    const int64_t m0 = static_cast<int64_t>(m_tile) * kBM;
    const int o0 = o_tile * kBN;
    const int b0 = o0;  // first row of the B tile
    const int nk = (A.d_in + kBK - 1) / kBK;

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

    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&A.tmx);
        prefetch_tensormap(&A.tmb);
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % kStages;
            if (kb >= kStages && !mbar_wait_bounded(&empty[s], ((kb / kStages) - 1) & 1, A.ew, 401))
                break;
            uint8_t* a = smem + s * kStageBytes;
            mbar_arrive_expect_tx(&full[s], kStageBytes);
            tma_load_2d(a, &A.tmx, &full[s], kb * kBK, static_cast<int32_t>(m0));
            tma_load_2d(a + kABytes, &A.tmb, &full[s], kb * kBK, b0);
        }
    } else if (warp == 1 && lane == 0) {
        constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, 0, 0);
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % kStages;
            if (!mbar_wait_bounded(&full[s], (kb / kStages) & 1, A.ew, 402)) break;
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
    mbar_wait_bounded(acc_full, 0, A.ew, 403);
    __syncwarp();
    tc_fence_after();

    // epilogue: thread = token row (TMEM lane quarter = warp % 4)
    const int lq = warp & 3;
    const int grp = warp >> 2;
    const int row = lq * 32 + lane;
    const int64_t t = m0 + row;
    const bool valid = t < A.N;
    const uint32_t trow = tmem + (static_cast<uint32_t>(lq * 32) << 16);
    const int nchunks = min(kBN, A.d_out - o0) / 16;
    if (kMode == kResidual) {
        // e = y - u leaves through shared memory: each warp group stages 32-column boxes of the
        // tile's 128 rows in the freed pipeline buffers (128-byte swizzle: 16-byte chunk j of
        // row i at position j ^ (i mod 8), conflict-free), and one thread of the group stores
        // each box with TMA (rows past N and columns past d_out are clipped).  The groups take
        // alternate boxes, two buffers each.  u is read one box ahead.
        const int nboxes = (nchunks + 1) / 2;
        const bool issuer = lq == 0 && lane == 0;
        auto group_sync = [grp]() {  // the group's four warps (barriers 1 and 2)
            if (grp == 0)
                named_bar_sync(1, 128);
            else
                named_bar_sync(2, 128);
        };
        const uint4* urow = reinterpret_cast<const uint4*>(A.u + (valid ? t * A.d_out + o0 : 0));
        uint4 un[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) un[h] = make_uint4(0u, 0u, 0u, 0u);
        if (valid && grp < nboxes) {
#pragma unroll
            for (int h = 0; h < 4; ++h)
                if (2 * grp + (h >> 1) < nchunks) un[h] = __ldg(urow + 4 * grp + h);
        }
        float sa = 0.f;
        int k = 0;
        for (int b = grp; b < nboxes; b += 2, ++k) {
            float* buf = reinterpret_cast<float*>(smem + (grp * 2 + (k & 1)) * kEBoxBytes);
            if (k >= 2) {
                // the store that last read this buffer (two boxes ago) is done with it
                if (issuer) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
                group_sync();
            }
            uint4 uc[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) uc[h] = un[h];
            if (valid && b + 2 < nboxes) {
#pragma unroll
                for (int h = 0; h < 4; ++h)
                    if (2 * (b + 2) + (h >> 1) < nchunks) un[h] = __ldg(urow + 4 * (b + 2) + h);
            }
#pragma unroll
            for (int hc = 0; hc < 2; ++hc) {
                const int c = 2 * b + hc;
                if (c >= nchunks) break;  // warp-uniform
                float v[16];
                tmem_ld16(trow + c * 16, v);
                tmem_wait_ld();
                float e[16];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint4 w = uc[2 * hc + h];
                    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        e[8 * h + 2 * q] = v[8 * h + 2 * q] - __uint_as_float(ww[q] << 16);
                        e[8 * h + 2 * q + 1] = v[8 * h + 2 * q + 1] - __uint_as_float(ww[q] & 0xFFFF0000u);
                    }
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float4 e4 = make_float4(e[4 * q], e[4 * q + 1], e[4 * q + 2], e[4 * q + 3]);
                    if (!valid) e4 = make_float4(0.f, 0.f, 0.f, 0.f);
                    sa = fmaf(e4.x, e4.x, sa);
                    sa = fmaf(e4.y, e4.y, sa);
                    sa = fmaf(e4.z, e4.z, sa);
                    sa = fmaf(e4.w, e4.w, sa);
                    const int j = (4 * hc + q) ^ (row & 7);
                    *reinterpret_cast<float4*>(buf + row * 32 + 4 * j) = e4;
                }
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            group_sync();
            if (issuer) {
                tma_store_2d(&A.tme, buf, o0 + 32 * b, static_cast<int32_t>(m0));
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            }
        }
        if (issuer) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        // the two groups' partial sums of a token, added in a fixed order
        if (grp == 1) red[row] = sa;
        __syncthreads();
        if (grp == 0 && valid) A.part_a[static_cast<int64_t>(o_tile) * A.N + t] = 0.5f * (sa + red[row]);
    } else {
        // the perturbed outputs of every draw; the two warp groups take alternate 16-column chunks
        for (int c = grp; c < nchunks; c += 2) {
            float v[16];
            tmem_ld16(trow + c * 16, v);
            tmem_wait_ld();
            if (!valid) continue;
            const uint32_t tg = A.key.token_offset + static_cast<uint32_t>(t);
            const uint32_t q0 = static_cast<uint32_t>((o0 + c * 16) >> 2) + A.key.quad_offset;
            for (int i = 0; i < A.K; ++i) {
                const int64_t at = (static_cast<int64_t>(i) * A.N + t) * A.ld_out + o0 + c * 16;
                float o[16];
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const F4 a = normal_quad(q0 + qq, tg, A.key.draw_offset + static_cast<uint32_t>(i),
                                             A.key.layer, A.key);
                    o[4 * qq] = fmaf(A.sigma, a.x, v[4 * qq]);
                    o[4 * qq + 1] = fmaf(A.sigma, a.y, v[4 * qq + 1]);
                    o[4 * qq + 2] = fmaf(A.sigma, a.z, v[4 * qq + 2]);
                    o[4 * qq + 3] = fmaf(A.sigma, a.w, v[4 * qq + 3]);
                }
                if (A.out_bf16) {
                    uint4 w[2];
                    uint32_t* wb = reinterpret_cast<uint32_t*>(w);
#pragma unroll
                    for (int h = 0; h < 8; ++h) {
                        __nv_bfloat162 b2 = __floats2bfloat162_rn(o[2 * h], o[2 * h + 1]);
                        wb[h] = *reinterpret_cast<uint32_t*>(&b2);
                    }
                    uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(A.y_out) + at);
                    dst[0] = w[0];
                    dst[1] = w[1];
                } else {
                    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(A.y_out) + at);
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq)
                        dst[qq] = make_float4(o[4 * qq], o[4 * qq + 1], o[4 * qq + 2], o[4 * qq + 3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------- persistent probe GEMM
// The probe mode as a persistent, warp-specialised kernel: one CTA per SM walks the tiles in the
// same order; warp 0 feeds a 4-stage TMA ring, warp 1 issues the MMAs into one of two
// 256-column accumulators, and warps 2-9 run the epilogue of the previous tile from the other
// accumulator meanwhile: warp w reads TMEM lanes 32 (w % 4) .. + 31 (its tokens) and the
// columns of half (w - 2) / 4 of the tile, so each (token, half) has its own partial sums.
constexpr int kPStages = 4;
constexpr int kPThreads = 320;  // producer, MMA issuer, eight epilogue warps
constexpr uint32_t kPSmemBytes = kPStages * kStageBytes + 1024 + 256;

__global__ void __launch_bounds__(kPThreads, 1) spsa_probe_gemm_kernel(const __grid_constant__ GemmArgs A) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kPStages * kStageBytes);
    uint64_t* empty = full + kPStages;
    uint64_t* acc_full = empty + kPStages;  // [2]
    uint64_t* acc_empty = acc_full + 2;     // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tiles = A.m_tiles * A.P * A.o_tiles;
    const int nk = (A.d_in + kBK - 1) / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 8);  // one arrival per epilogue warp
        }
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 2 * kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tensormap(&A.tmx);
            prefetch_tensormap(&A.tmb);
            uint32_t kc = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
                const int m_tile = tile % A.m_tiles;
                const int j = (tile / A.m_tiles) % A.P;
                const int o_tile = tile / (A.m_tiles * A.P);
                const int b0 = (j * A.o_tiles + o_tile) * kBN;
                for (int kb = 0; kb < nk; ++kb, ++kc) {
                    const int s = kc % kPStages;
                    if (kc >= kPStages &&
                        !mbar_wait_bounded(&empty[s], ((kc / kPStages) - 1) & 1, A.ew, 411)) {
                        ok = false;
                        break;
                    }
                    uint8_t* a = smem + s * kStageBytes;
                    mbar_arrive_expect_tx(&full[s], kStageBytes);
                    tma_load_2d(a, &A.tmx, &full[s], kb * kBK, m_tile * kBM);
                    tma_load_2d(a + kABytes, &A.tmb, &full[s], kb * kBK, b0);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, 0, 0);
            uint32_t kc = 0;
            int lt = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++lt) {
                const int buf = lt & 1;
                // the epilogue of the tile that last used this accumulator has read it
                if (lt >= 2 && !mbar_wait_bounded(&acc_empty[buf], ((lt >> 1) - 1) & 1, A.ew, 412))
                    break;
                tc_fence_after();
                const uint32_t d = tmem + static_cast<uint32_t>(buf * kTmemCols);
                for (int kb = 0; kb < nk; ++kb, ++kc) {
                    const int s = kc % kPStages;
                    if (!mbar_wait_bounded(&full[s], (kc / kPStages) & 1, A.ew, 413)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + s * kStageBytes);
                    const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint64_t ad = sdesc_sw128(a_addr + kk * 32, 16, 1024);
                        const uint64_t bd = sdesc_sw128(b_addr + kk * 32, 16, 1024);
                        umma_bf16(d, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    umma_commit(&empty[s]);
                }
                umma_commit(&acc_full[buf]);
            }
        }
    } else {
        // epilogue warps 2..9: TMEM lane quarter q = warp % 4, column half hf
        const int q = warp & 3;
        const int hf = (warp - 2) >> 2;
        int lt = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++lt) {
            const int buf = lt & 1;
            const int m_tile = tile % A.m_tiles;
            const int j = (tile / A.m_tiles) % A.P;
            const int o_tile = tile / (A.m_tiles * A.P);
            const int o0 = o_tile * kBN;
            if (!mbar_wait_bounded(&acc_full[buf], (lt >> 1) & 1, A.ew, 414)) break;
            __syncwarp();
            tc_fence_after();
            const int row = q * 32 + lane;
            const int64_t t = static_cast<int64_t>(m_tile) * kBM + row;
            const bool valid = t < A.N;
            const uint32_t trow = tmem + static_cast<uint32_t>(buf * kTmemCols) +
                                  (static_cast<uint32_t>(q * 32) << 16);
            const int nchunks = min(kBN, A.d_out - o0) / 16;
            const int c_end = min(nchunks, (hf + 1) * (kBN / 32));
            float sa = 0.f, sb = 0.f;
            for (int c = hf * (kBN / 32); c < c_end; ++c) {
                float v[16];
                tmem_ld16(trow + c * 16, v);
                tmem_wait_ld();
                if (!valid) continue;
                const float4* e4 = reinterpret_cast<const float4*>(A.e + t * A.d_out + o0 + c * 16);
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const float4 e = __ldg(e4 + qq);
                    sa = fmaf(e.x, v[4 * qq], sa);
                    sa = fmaf(e.y, v[4 * qq + 1], sa);
                    sa = fmaf(e.z, v[4 * qq + 2], sa);
                    sa = fmaf(e.w, v[4 * qq + 3], sa);
                    sb = fmaf(v[4 * qq], v[4 * qq], sb);
                    sb = fmaf(v[4 * qq + 1], v[4 * qq + 1], sb);
                    sb = fmaf(v[4 * qq + 2], v[4 * qq + 2], sb);
                    sb = fmaf(v[4 * qq + 3], v[4 * qq + 3], sb);
                }
            }
            // the accumulator may be refilled once every epilogue warp has read it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);
            if (valid) {
                const int64_t slot = (static_cast<int64_t>(j) * A.o_tiles + o_tile) * 2 + hf;
                A.part_a[slot * A.N + t] = sa;
                A.part_b[slot * A.N + t] = sb;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 2 * kTmemCols);
}

// ---------------------------------------------------------------- reductions
// Stage 1: block (slot, chunk) sums its chunk of tokens of one partial row in a fixed order
// (per thread in token order, then the threads in a fixed tree).  Slots: 2 P o_tiles rows of
// <e, v> (probe, output tile, column half), then as many of |v|^2, then o_tiles rows of
// 1/2 |e|^2.
constexpr int kRedChunk = 4096;
__global__ void __launch_bounds__(256) spsa_reduce_kernel(const float* part_ev, const float* part_vv,
                                                          const float* part_l0, int64_t N,
                                                          int n_pv, int o_tiles, int n_chunks,
                                                          float* sums) {
    __shared__ float sh[256];
    const int slot = blockIdx.x / n_chunks, chunk = blockIdx.x % n_chunks;
    const float* row = slot < n_pv ? part_ev + static_cast<int64_t>(slot) * N
                       : slot < 2 * n_pv ? part_vv + static_cast<int64_t>(slot - n_pv) * N
                                         : part_l0 + static_cast<int64_t>(slot - 2 * n_pv) * N;
    const int64_t t_end = min(N, static_cast<int64_t>(chunk + 1) * kRedChunk);
    float a = 0.f;
    for (int64_t t = static_cast<int64_t>(chunk) * kRedChunk + threadIdx.x; t < t_end; t += 256)
        a += row[t];
    sh[threadIdx.x] = a;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (threadIdx.x < w) sh[threadIdx.x] += sh[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) sums[blockIdx.x] = sh[0];
}

// Stage 2: one thread per probe adds its tiles' chunk sums in order; p, L_+, L_-.
__global__ void spsa_finish_kernel(const float* sums, int P, int o_tiles, int n_chunks, float eps,
                                   float* p, float* Lp, float* Lm) {
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= P) return;
    const int n_pv = P * o_tiles * 2;  // (probe, output tile, column half) slots
    float ev = 0.f, vv = 0.f, l0 = 0.f;
    for (int ot = 0; ot < o_tiles; ++ot) {
        for (int h = 0; h < 2; ++h)
            for (int c = 0; c < n_chunks; ++c) {
                const int64_t sl = (static_cast<int64_t>(j) * o_tiles + ot) * 2 + h;
                ev += sums[sl * n_chunks + c];
                vv += sums[(n_pv + sl) * n_chunks + c];
            }
        for (int c = 0; c < n_chunks; ++c)
            l0 += sums[(static_cast<int64_t>(2 * n_pv + ot)) * n_chunks + c];
    }
    p[j] = ev;  // (L_+ - L_-) / (2 eps) = sum_t <e_t, v_t>
    const float curv = 0.5f * eps * eps * vv;
    if (Lp) Lp[j] = l0 + eps * ev + curv;
    if (Lm) Lm[j] = l0 - eps * ev + curv;
}

// G[o][k] (+)= scale * sum_j p_j z_j[o][k]: one thread per (o, channel quad), probes in order.
__global__ void __launch_bounds__(256) spsa_estimate_kernel(const __grid_constant__ NoiseKey key,
                                                            const float* __restrict__ p, int P,
                                                            int d_out, int d_in, float scale,
                                                            float* G, int accumulate,
                                                            uint64_t nq_magic) {
    const int nq = d_in >> 2;
    const int64_t total = static_cast<int64_t>(d_out) * nq;
    for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int o = static_cast<int>(div_by_magic(idx, nq, nq_magic));
        const int q = static_cast<int>(idx - static_cast<int64_t>(o) * nq);
        F2 a02{0.f, 0.f}, a13{0.f, 0.f};  // channels (4q, 4q+2) and (4q+1, 4q+3)
        const PhiloxRun run = philox_run_over_word2(static_cast<uint32_t>(q), static_cast<uint32_t>(o),
                                                    key.layer | kWeightSpace, key);
        // unrolled so that independent Philox chains of consecutive probes interleave
#pragma unroll 4
        for (int j = 0; j < P; ++j) {
            const float pj = __ldg(p + j);
            const PolarPairs z = box_muller_pairs(
                philox_word2(key.draw_offset + static_cast<uint32_t>(j), run, key));
            const F2 r = mul2(F2{kKappa, kKappa}, z.nq);
            const F2 zc = mul2(r, z.c), zs = mul2(r, z.s);
            // the direction is the bf16 value of the normal
            const __nv_bfloat162 bc = __floats2bfloat162_rn(zc.x, zc.y);
            const __nv_bfloat162 bs = __floats2bfloat162_rn(zs.x, zs.y);
            a02 = fma2(F2{pj, pj}, F2{__low2float(bc), __high2float(bc)}, a02);
            a13 = fma2(F2{pj, pj}, F2{__low2float(bs), __high2float(bs)}, a13);
        }
        float4* g = reinterpret_cast<float4*>(G + static_cast<int64_t>(o) * d_in + 4 * q);
        float4 r = make_float4(scale * a02.x, scale * a13.x, scale * a02.y, scale * a13.y);
        if (accumulate) {
            const float4 old = *g;
            r.x += old.x;
            r.y += old.y;
            r.z += old.z;
            r.w += old.w;
        }
        *g = r;
    }
}

}  // namespace

size_t spsa_workspace_bytes(int64_t N, int32_t d_in, int32_t d_out, int32_t P) {
    const int o_tiles = pad256(d_out) / kBN;
    return align_up(static_cast<size_t>(P) * pad256(d_out) * d_in * 2, 256) +  // Z
           align_up(static_cast<size_t>(N) * d_out * 4, 256) +                    // e
           align_up(static_cast<size_t>(o_tiles) * N * 4, 256) +                  // 1/2 |e|^2
           2 * align_up(static_cast<size_t>(2 * P) * o_tiles * N * 4, 256) +      // <e,v>, |v|^2
           align_up(static_cast<size_t>(4 * P + 1) * o_tiles * ((N + 4095) / 4096) * 4, 256);
}

dust_status spsa_probe_launch(const void* x, const void* W, const void* u, int64_t N, int32_t d_in,
                              int32_t d_out, int32_t P, float eps, NoiseKey key, float* p,
                              float* Lp, float* Lm, void* ws, cudaStream_t s) {
    const int dpad = pad256(d_out);
    const int o_tiles = dpad / kBN;
    const int m_tiles = static_cast<int>((N + kBM - 1) / kBM);
    if (static_cast<int64_t>(m_tiles) * o_tiles * P > 2147483647LL) return DUST_ERR_UNSUPPORTED;
    char* w = static_cast<char*>(ws);
    __nv_bfloat16* Z = reinterpret_cast<__nv_bfloat16*>(w);
    w += align_up(static_cast<size_t>(P) * dpad * d_in * 2, 256);
    float* e = reinterpret_cast<float*>(w);
    w += align_up(static_cast<size_t>(N) * d_out * 4, 256);
    float* pl0 = reinterpret_cast<float*>(w);
    w += align_up(static_cast<size_t>(o_tiles) * N * 4, 256);
    float* pev = reinterpret_cast<float*>(w);
    w += align_up(static_cast<size_t>(2 * P) * o_tiles * N * 4, 256);
    float* pvv = reinterpret_cast<float*>(w);
    w += align_up(static_cast<size_t>(2 * P) * o_tiles * N * 4, 256);
    float* sums = reinterpret_cast<float*>(w);

    GemmArgs R{};
    R.u = static_cast<const __nv_bfloat16*>(u);
    R.e = e;
    R.part_a = pl0;
    R.part_b = nullptr;
    R.ew = device_error_word();
    R.N = N;
    R.d_in = d_in;
    R.d_out = d_out;
    R.o_tiles = o_tiles;
    R.P = P;
    R.m_tiles = m_tiles;
    if (!make_tmap_bf16_2d(&R.tmx, x, static_cast<uint64_t>(N), d_in, kBM, kBK) ||
        !make_tmap_bf16_2d(&R.tmb, W, static_cast<uint64_t>(d_out), d_in, kBN, kBK) ||
        !make_tmap_f32_2d_sw128(&R.tme, e, static_cast<uint64_t>(N), d_out, d_out, kBM))
        return DUST_ERR_CUDA;
    GemmArgs Q = R;
    Q.part_a = pev;
    Q.part_b = pvv;
    if (!make_tmap_bf16_2d(&Q.tmb, Z, static_cast<uint64_t>(P) * dpad, d_in, kBN, kBK))
        return DUST_ERR_CUDA;
    if (cudaFuncSetAttribute(spsa_gemm_kernel<kResidual>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes)) != cudaSuccess ||
        cudaFuncSetAttribute(spsa_probe_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kPSmemBytes)) != cudaSuccess)
        return DUST_ERR_CUDA;
    const int64_t dir_rows = static_cast<int64_t>(P) * dpad;  // one warp each, 8 per block
    prof_begin(s);
    spsa_dir_kernel<<<static_cast<unsigned>(std::min<int64_t>((dir_rows + 7) / 8,
                                                              static_cast<int64_t>(num_sms()) * 8)),
                      256, 0, s>>>(key, P, d_out, dpad, d_in, Z);
    prof_end(s, "spsa_directions");
    prof_begin(s);
    spsa_gemm_kernel<kResidual><<<static_cast<unsigned>(m_tiles * o_tiles), kThreads, kSmemBytes, s>>>(R);
    prof_end(s, "spsa_residual_gemm");
    prof_begin(s);
    const int64_t probe_tiles = static_cast<int64_t>(m_tiles) * o_tiles * P;
    spsa_probe_gemm_kernel<<<static_cast<unsigned>(std::min<int64_t>(probe_tiles, num_sms())),
                             kPThreads, kPSmemBytes, s>>>(Q);
    prof_end(s, "spsa_probe_gemm");
    const int n_chunks = static_cast<int>((N + kRedChunk - 1) / kRedChunk);
    const int n_pv = 2 * P * o_tiles;
    prof_begin(s);
    spsa_reduce_kernel<<<static_cast<unsigned>((2 * n_pv + o_tiles) * n_chunks), 256, 0, s>>>(
        pev, pvv, pl0, N, n_pv, o_tiles, n_chunks, sums);
    spsa_finish_kernel<<<static_cast<unsigned>((P + 127) / 128), 128, 0, s>>>(sums, P, o_tiles,
                                                                            n_chunks, eps, p, Lp, Lm);
    prof_end(s, "spsa_reduce");
    return cudaGetLastError() == cudaSuccess ? DUST_OK : DUST_ERR_CUDA;
}

dust_status noisy_output_launch(const void* x, const void* W, int64_t N, int32_t d_in,
                               int32_t d_out, int32_t K, float sigma, NoiseKey key, void* y_out,
                               int out_bf16, int64_t ld_out, cudaStream_t s) {
    GemmArgs G{};
    G.y_out = y_out;
    G.ew = device_error_word();
    G.N = N;
    G.ld_out = ld_out;
    G.d_in = d_in;
    G.d_out = d_out;
    G.o_tiles = pad256(d_out) / kBN;
    G.P = 1;
    G.m_tiles = static_cast<int>((N + kBM - 1) / kBM);
    G.K = K;
    G.out_bf16 = out_bf16;
    G.sigma = sigma;
    G.key = key;
    if (!make_tmap_bf16_2d(&G.tmx, x, static_cast<uint64_t>(N), d_in, kBM, kBK) ||
        !make_tmap_bf16_2d(&G.tmb, W, static_cast<uint64_t>(d_out), d_in, kBN, kBK))
        return DUST_ERR_CUDA;
    if (cudaFuncSetAttribute(spsa_gemm_kernel<kNoisyOut>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes)) != cudaSuccess)
        return DUST_ERR_CUDA;
    prof_begin(s);
    spsa_gemm_kernel<kNoisyOut><<<static_cast<unsigned>(G.m_tiles * G.o_tiles), kThreads,
                                  kSmemBytes, s>>>(G);
    prof_end(s, "noisy_linear_output");
    return cudaGetLastError() == cudaSuccess ? DUST_OK : DUST_ERR_CUDA;
}

dust_status spsa_estimate_launch(const float* p, int32_t P, int32_t P_total, int32_t d_in,
                                 int32_t d_out, NoiseKey key, float* G, int accumulate,
                                 cudaStream_t s) {
    const int64_t total = static_cast<int64_t>(d_out) * (d_in / 4);
    prof_begin(s);
    spsa_estimate_kernel<<<static_cast<unsigned>(std::min<int64_t>((total + 255) / 256,
                                                                   static_cast<int64_t>(num_sms()) * 16)),
                           256, 0, s>>>(key, p, P, d_out, d_in, 1.0f / static_cast<float>(P_total),
                                        G, accumulate, div_magic(d_in / 4));
    prof_end(s, "spsa_estimate");
    return cudaGetLastError() == cudaSuccess ? DUST_OK : DUST_ERR_CUDA;
}

}  // namespace dust
