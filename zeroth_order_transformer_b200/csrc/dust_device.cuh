// Device-side building blocks shared by the libdust kernels: the counter-based noise
// generator, bounded waits, and thin wrappers over the sm_100a PTX used by the tensor-core
// kernels (mbarrier, TMA, tcgen05).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dust_internal.h"

namespace dust {

// ----------------------------------------------------------------------------------------
// Device error word: one per device, written by kernels whose bounded wait ran out.
// ----------------------------------------------------------------------------------------
enum DeviceError : int { kDevOk = 0, kDevTimeout = 4 };

struct ErrorWord {
    int code;
    int info;
};

__device__ __forceinline__ void report_error(ErrorWord* ew, int code, int info) {
    if (ew && atomicCAS(&ew->code, 0, code) == 0) atomicExch(&ew->info, info);
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded waits give up after this many nanoseconds.
constexpr uint64_t kWaitLimitNs = 1000000000ull;

// ----------------------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11): 10 rounds; each multiplies counter
// words 0 and 2 by the two round multipliers into 64-bit products and forms
// (hi1 ^ c1 ^ key0, lo1, hi0 ^ c3 ^ key1, lo0).  The round keys come precomputed in
// NoiseKey::rk (parameter space), so each round is two widening multiplies and two
// three-input XORs.
// ----------------------------------------------------------------------------------------
constexpr uint32_t kPhiloxM0 = 0xD2511F53u;
constexpr uint32_t kPhiloxM1 = 0xCD9E8D57u;

struct U4 {
    uint32_t x, y, z, w;
};

__device__ __forceinline__ U4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                            const NoiseKey& key) {
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        const uint64_t p0 = static_cast<uint64_t>(kPhiloxM0) * c0;
        const uint64_t p1 = static_cast<uint64_t>(kPhiloxM1) * c2;
        const uint32_t n0 = static_cast<uint32_t>(p1 >> 32) ^ c1 ^ key.rk[2 * round];
        const uint32_t n2 = static_cast<uint32_t>(p0 >> 32) ^ c3 ^ key.rk[2 * round + 1];
        c1 = static_cast<uint32_t>(p1);
        c3 = static_cast<uint32_t>(p0);
        c0 = n0;
        c2 = n2;
    }
    return U4{c0, c1, c2, c3};
}

// Runs of blocks whose counters differ in one word only.  The noise kernels walk either the
// channel quads of one (token, draw, layer) (word 0 varies) or the draws of one (quad, token,
// layer) (word 2 varies).  Then the first round's product of the fixed multiplied word and
// the second round's product of the word it produces are the same for the whole run: they are
// formed once, with the round keys and fixed words that are XORed into them, and each block of
// the run costs 18 widening multiplies instead of 20.  The words are those of philox4x32_10.
//
// Word 0 varies, counter (q, c1, c2, c3):
//   round 0:  (hi(M1 c2) ^ c1 ^ rk0,  lo(M1 c2),  hi(M0 q) ^ c3 ^ rk1,  lo(M0 q))
//             = (a, b, hi(M0 q) ^ e, lo(M0 q))              a, b, e = c3 ^ rk1 fixed
//   round 1:  (hi(M1 x2) ^ b ^ rk2,  lo(M1 x2),  hi(M0 a) ^ x3 ^ rk3,  lo(M0 a))
//             = (hi(M1 x2) ^ f, lo(M1 x2), h ^ x3, d)       f = b ^ rk2, h = hi(M0 a) ^ rk3, d fixed
// Word 2 varies, counter (c0, c1, i, c3):
//   round 0:  (hi(M1 i) ^ g,  lo(M1 i),  E,  F)             g = c1 ^ rk0; E = hi(M0 c0) ^ c3 ^ rk1,
//                                                           F = lo(M0 c0) fixed
//   round 1:  (hi(M1 E) ^ x1 ^ rk2,  lo(M1 E),  hi(M0 x0) ^ F ^ rk3,  lo(M0 x0))
//             = (h ^ x1, H, hi(M0 x0) ^ f, lo(M0 x0))       h = hi(M1 E) ^ rk2, H, f = F ^ rk3 fixed
struct PhiloxRun {
    uint32_t k1, k2, k3, k4;  // word 0 varies: e, f, h, d;  word 2 varies: g, h, H, f
};

__device__ __forceinline__ void philox_rounds_2_to_9(uint32_t& c0, uint32_t& c1, uint32_t& c2,
                                                     uint32_t& c3, const NoiseKey& key) {
#pragma unroll
    for (int round = 2; round < 10; ++round) {
        const uint64_t p0 = static_cast<uint64_t>(kPhiloxM0) * c0;
        const uint64_t p1 = static_cast<uint64_t>(kPhiloxM1) * c2;
        const uint32_t n0 = static_cast<uint32_t>(p1 >> 32) ^ c1 ^ key.rk[2 * round];
        const uint32_t n2 = static_cast<uint32_t>(p0 >> 32) ^ c3 ^ key.rk[2 * round + 1];
        c1 = static_cast<uint32_t>(p1);
        c3 = static_cast<uint32_t>(p0);
        c0 = n0;
        c2 = n2;
    }
}

__device__ __forceinline__ PhiloxRun philox_run_over_word0(uint32_t c1, uint32_t c2, uint32_t c3,
                                                           const NoiseKey& key) {
    const uint64_t p1 = static_cast<uint64_t>(kPhiloxM1) * c2;
    const uint32_t a = static_cast<uint32_t>(p1 >> 32) ^ c1 ^ key.rk[0];
    const uint64_t pa = static_cast<uint64_t>(kPhiloxM0) * a;
    return PhiloxRun{c3 ^ key.rk[1], static_cast<uint32_t>(p1) ^ key.rk[2],
                     static_cast<uint32_t>(pa >> 32) ^ key.rk[3], static_cast<uint32_t>(pa)};
}

__device__ __forceinline__ U4 philox_word0(uint32_t q, const PhiloxRun& R, const NoiseKey& key) {
    const uint64_t p0 = static_cast<uint64_t>(kPhiloxM0) * q;
    const uint32_t x2 = static_cast<uint32_t>(p0 >> 32) ^ R.k1;
    const uint32_t x3 = static_cast<uint32_t>(p0);
    const uint64_t p1 = static_cast<uint64_t>(kPhiloxM1) * x2;
    uint32_t c0 = static_cast<uint32_t>(p1 >> 32) ^ R.k2;
    uint32_t c1 = static_cast<uint32_t>(p1);
    uint32_t c2 = R.k3 ^ x3;
    uint32_t c3 = R.k4;
    philox_rounds_2_to_9(c0, c1, c2, c3, key);
    return U4{c0, c1, c2, c3};
}

__device__ __forceinline__ PhiloxRun philox_run_over_word2(uint32_t c0, uint32_t c1, uint32_t c3,
                                                           const NoiseKey& key) {
    const uint64_t p0 = static_cast<uint64_t>(kPhiloxM0) * c0;
    const uint32_t E = static_cast<uint32_t>(p0 >> 32) ^ c3 ^ key.rk[1];
    const uint64_t pE = static_cast<uint64_t>(kPhiloxM1) * E;
    return PhiloxRun{c1 ^ key.rk[0], static_cast<uint32_t>(pE >> 32) ^ key.rk[2],
                     static_cast<uint32_t>(pE), static_cast<uint32_t>(p0) ^ key.rk[3]};
}

__device__ __forceinline__ U4 philox_word2(uint32_t i, const PhiloxRun& R, const NoiseKey& key) {
    const uint64_t p1 = static_cast<uint64_t>(kPhiloxM1) * i;
    const uint32_t x0 = static_cast<uint32_t>(p1 >> 32) ^ R.k1;
    const uint32_t x1 = static_cast<uint32_t>(p1);
    const uint64_t p0 = static_cast<uint64_t>(kPhiloxM0) * x0;
    uint32_t c0 = R.k2 ^ x1;
    uint32_t c1 = R.k3;
    uint32_t c2 = static_cast<uint32_t>(p0 >> 32) ^ R.k4;
    uint32_t c3 = static_cast<uint32_t>(p0);
    philox_rounds_2_to_9(c0, c1, c2, c3, key);
    return U4{c0, c1, c2, c3};
}

// The float with the given sign and exponent bits and the word's top 23 bits m = w >> 9 as
// mantissa (written as an add: the two bit fields do not overlap).
__device__ __forceinline__ float mantissa_float(uint32_t exp_bits, uint32_t w) {
    return __uint_as_float(exp_bits + (w >> 9));
}

// Hardware approximations (PTX .approx with flush-to-zero; every input here is a normal
// float): base-2 logarithm, reciprocal square root, sine and cosine in radians.
__device__ __forceinline__ float lg2_approx(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rsqrt_approx(float x) {
    float y;
    asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float sin_approx(float x) {
    float y;
    asm("sin.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float cos_approx(float x) {
    float y;
    asm("cos.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// y = -log2 u for u in [2^-24, 1 - 2^-24], from the hardware base-2 logarithm.  Its small
// absolute error is amplified in q = sqrt(y) by 1 / (2 q), which matters only for u close to
// 1; there (u > 1 - 2^-10) the Taylor series -log2(1 - v) = (v + v^2/2 + v^3/3 + ...) / ln 2
// in the exact v = 1 - u replaces it (the omitted terms are below v^3 / 4 relative, i.e.
// under 2^-32).
__device__ __forceinline__ float neg_lg2_near_one(float u, float y_fast) {
    if (u > 0.9990234375f) {
        const float v = 1.0f - u;
        return v * fmaf(v, fmaf(v, 0.48089834696298783f, 0.72134752044448170f),
                        1.4426950408889634f);  // 1/(3 ln 2), 1/(2 ln 2), 1/ln 2
    }
    return y_fast;
}
// Words whose uniform exceeds 1 - 2^-10 have their top ten bits set.
constexpr uint32_t kNearOneWord = 0xFFC00000u;

// rho = sqrt(-2 ln u) = kKappa sqrt(-log2 u), kKappa = sqrt(2 ln 2).
constexpr float kKappa = 1.1774100225154747f;

struct F4 {
    float x, y, z, w;
};

// Two-wide fp32 arithmetic: sm_100's packed f32x2 instructions do two independent,
// correctly rounded operations (the same results as two scalar ones) in one issue slot.
struct F2 {
    float x, y;
};
__device__ __forceinline__ F2 fma2(F2 a, F2 b, F2 c) {
    F2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ F2 mul2(F2 a, F2 b) {
    F2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ F2 add2(F2 a, F2 b) {
    F2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// Box-Muller on one Philox block in scaled polar form, as packed pairs: pair p (words 2p,
// 2p+1) has the radius word's L_p = log2 u(w_2p) <= 0, so y_p = -L_p and q_p = sqrt(y_p) (the
// radius is rho_p = kKappa q_p, rho_p^2 = 2 ln 2 y_p), and the angle 2 pi u(w_2p+1) - pi, where
// the hardware sine and cosine keep their absolute error bound.  The -pi shift flips both
// signs, so
//     z_2p = -kKappa q_p cos_p = kKappa nq_p cos_p,   z_2p+1 = kKappa nq_p sin_p,
// with nq_p = -q_p = L_p rsqrt(-L_p).  Lane x of each pair is pair 0 (channels 4q, 4q+1),
// lane y pair 1 (channels 4q+2, 4q+3).  Consumers fold kKappa (and 2 ln 2) into their own
// coefficients.
struct PolarPairs {
    F2 L;   // log2 u of the radius words
    F2 nq;  // -sqrt(-L)
    F2 c;   // cosines of the two angles
    F2 s;   // sines
};

__device__ __forceinline__ PolarPairs box_muller_pairs(const U4& w) {
    // u(w) = (2m + 1) 2^-24 with m = w >> 9, exact: 1 + m 2^-23 (exponent 0, mantissa m) minus
    // 1 - 2^-24 leaves (2m + 1) 2^-24, which fits in 24 bits; both radius words at once
    const F2 u = add2(F2{mantissa_float(0x3f800000u, w.x), mantissa_float(0x3f800000u, w.z)},
                      F2{-0.99999994f, -0.99999994f});
    PolarPairs p;
    p.L.x = lg2_approx(u.x);
    p.L.y = lg2_approx(u.y);
    if (max(w.x, w.z) >= kNearOneWord) {  // rare: about 1 block in 500
        p.L.x = -neg_lg2_near_one(u.x, -p.L.x);
        p.L.y = -neg_lg2_near_one(u.y, -p.L.y);
    }
    p.nq = mul2(p.L, F2{rsqrt_approx(-p.L.x), rsqrt_approx(-p.L.y)});
    // Box-Muller angle shifted by -pi, one FMA per angle word: the float f = 2 + m 2^-22
    // (exponent 1, mantissa m) gives 2 pi u(w) - pi = pi f - 3 pi + 2 pi 2^-24, which lies in
    // [-pi, pi) (largest error over all m: 3.5e-7 rad)
    const F2 a = fma2(F2{3.14159265358979323846f, 3.14159265358979323846f},
                      F2{mantissa_float(0x40000000u, w.y), mantissa_float(0x40000000u, w.w)},
                      F2{-9.4247775872730683f, -9.4247775872730683f});  // -3 pi + 2 pi 2^-24
    p.c = F2{cos_approx(a.x), cos_approx(a.y)};
    p.s = F2{sin_approx(a.x), sin_approx(a.y)};
    return p;
}

// The same block with scalar fields: y_p = -L_p >= 0 and q_p = sqrt(y_p).
struct Polar4 {
    float y0, q0, c0, s0;  // pair 0: channels 4q, 4q+1
    float y1, q1, c1, s1;  // pair 1: channels 4q+2, 4q+3
};

__device__ __forceinline__ Polar4 box_muller_polar(const U4& w) {
    const PolarPairs p = box_muller_pairs(w);
    return Polar4{-p.L.x, -p.nq.x, p.c.x, p.s.x, -p.L.y, -p.nq.y, p.c.y, p.s.y};
}

__device__ __forceinline__ Polar4 normal_quad_polar(uint32_t q, uint32_t t, uint32_t i,
                                                    uint32_t layer, const NoiseKey& key) {
    return box_muller_polar(philox4x32_10(q, t, i, layer, key));
}

// The four normals a[4q .. 4q+3] of (token, draw, layer).
__device__ __forceinline__ F4 normal_quad(uint32_t q, uint32_t t, uint32_t i, uint32_t layer,
                                          const NoiseKey& key) {
    const Polar4 p = normal_quad_polar(q, t, i, layer, key);
    const float r0 = -kKappa * p.q0, r1 = -kKappa * p.q1;
    return F4{r0 * p.c0, r0 * p.s0, r1 * p.c1, r1 * p.s1};
}

// ----------------------------------------------------------------------------------------
// Optimizer step on one element of the weight estimate g (decoupled weight decay first):
//   SGD with momentum:  m <- mu m + g;  w <- w - lr m
//   Adam (bias-corrected): m <- b1 m + (1-b1) g;  v <- b2 v + (1-b2) g^2;
//                          w <- w - lr (m / c1) / (sqrt(v / c2) + eps),  c = 1 - beta^t
// ----------------------------------------------------------------------------------------
__device__ __forceinline__ void opt_update(const OptParams& o, float g, float& w, float& m,
                                           float& v) {
    w = fmaf(-o.lr_wd, w, w);
    if (o.kind == DUST_OPT_SGD_MOMENTUM) {
        m = fmaf(o.mu, m, g);
        w = fmaf(-o.lr, m, w);
    } else {
        m = fmaf(o.b1, m, o.omb1 * g);
        v = fmaf(o.b2, v, o.omb2 * (g * g));
        w = w - o.lr * (m / o.c1) / (sqrtf(v / o.c2) + o.eps);
    }
}

// Applies the step to 4 consecutive elements at index e (a multiple of 4) of the targets.
__device__ __forceinline__ void opt_update4(const OptParams& o, const OptTargets& t, int64_t e,
                                            float4 g) {
    float4 w = *reinterpret_cast<const float4*>(t.W + e);
    float4 m = *reinterpret_cast<const float4*>(t.m + e);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (o.kind == DUST_OPT_ADAM) v = *reinterpret_cast<const float4*>(t.v + e);
    opt_update(o, g.x, w.x, m.x, v.x);
    opt_update(o, g.y, w.y, m.y, v.y);
    opt_update(o, g.z, w.z, m.z, v.z);
    opt_update(o, g.w, w.w, m.w, v.w);
    *reinterpret_cast<float4*>(t.W + e) = w;
    *reinterpret_cast<float4*>(t.m + e) = m;
    if (o.kind == DUST_OPT_ADAM) *reinterpret_cast<float4*>(t.v + e) = v;
    if (t.W_bf16) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(w.x, w.y);
        __nv_bfloat162 hi = __floats2bfloat162_rn(w.z, w.w);
        uint2 b;
        b.x = *reinterpret_cast<uint32_t*>(&lo);
        b.y = *reinterpret_cast<uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(t.W_bf16) + e) = b;
    }
}

// ----------------------------------------------------------------------------------------
// Shared-memory addresses, mbarriers, TMA.
// ----------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for phase `parity` of `bar`; gives up after kWaitLimitNs, reports `site` and
// returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, ErrorWord* ew,
                                                  int site) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            report_error(ew, kDevTimeout, site);
            return false;
        }
    }
}

// The same for waits expected to be long, by warps that share their SM with busy ones: sleeps
// `ns` between polls so that the waiting warp takes few issue slots.
__device__ __forceinline__ bool mbar_wait_bounded_sleep(uint64_t* bar, uint32_t parity, ErrorWord* ew,
                                                        int site, uint32_t ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        __nanosleep(ns);
        if (mbar_try_wait(bar, parity)) return true;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            report_error(ew, kDevTimeout, site);
            return false;
        }
    }
}

// 2-D tiled TMA load of box (x, y) into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map,
                                            uint64_t* bar, int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// 2-D tiled TMA store of box (x, y) from shared memory, tracked by the thread's bulk group.
// Elements outside the tensor are not written.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* smem_src,
                                             int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(smem_u32(smem_src)), "r"(x), "r"(y)
        : "memory");
}

// Barrier `id` (1 .. 15; 0 is __syncthreads) over `n` threads (a multiple of 32).
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ----------------------------------------------------------------------------------------
// tcgen05: tensor memory allocation, MMA issue, commit, and TMEM <-> register moves.
// ----------------------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem], bf16 inputs, fp32 accumulator (kind::f16).
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once every previously issued tcgen05.mma of this thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// Instruction descriptor of kind::f16 with bf16 A/B, fp32 D, M x N tile; a_mn / b_mn select
// MN-major (1) or K-major (0) operands.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn, int b_mn) {
    return (1u << 4)                              // D format: f32
           | (1u << 7)                            // A format: bf16
           | (1u << 10)                           // B format: bf16
           | (static_cast<uint32_t>(a_mn) << 15)  // A major
           | (static_cast<uint32_t>(b_mn) << 16)  // B major
           | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand (version 1, base offset 0;
// tiles are 1024-byte aligned).  lbo / sbo are byte offsets (multiples of 16).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;  // descriptor version for tcgen05
    d |= static_cast<uint64_t>(2) << 61;  // 128-byte swizzle
    return d;
}

// 32 lanes x 16 columns of 32-bit TMEM words: thread `lane` of the warp gets the 16 columns
// of TMEM lane (warp_quarter * 32 + lane).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15]))
        : "memory");
}

// 32 lanes x 8 columns: thread `lane` gets 8 columns of TMEM lane (warp_quarter * 32 + lane).
// The registers are not valid until tmem_wait_ld8 on the same array.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = __uint_as_float(r[j]);
}
// Waits for this thread's outstanding TMEM loads; the array is passed through the asm so that
// no read of it is scheduled before the wait.
__device__ __forceinline__ void tmem_wait_ld8(float (&v)[8]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]),
                   "+f"(v[6]), "+f"(v[7])
                 :
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

}  // namespace dust
