// Optimizer step on a weight estimate (Dust review page, section "설정": the estimate drives
// SGD with momentum; section "Adam에서도 통할까?": the same estimate fed to Adam).  An
// elementwise, HBM-bound pass: per element it reads g, w, m (and v) and writes w, m (and v),
// plus an optional bf16 copy of w for the next forward.
#include <algorithm>
#include <cmath>

#include "dust_device.cuh"
#include "dust_internal.h"

namespace dust {
namespace {

__global__ void opt_step_kernel(const OptParams o, const float* __restrict__ G, const OptTargets t,
                                int64_t n) {
    const int64_t n4 = n / 4;
    for (int64_t q = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; q < n4;
         q += static_cast<int64_t>(gridDim.x) * blockDim.x)
        opt_update4(o, t, 4 * q, __ldg(reinterpret_cast<const float4*>(G) + q));
    // tail (n not a multiple of 4)
    const int64_t e = 4 * n4 + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (blockIdx.x == 0 && e < n) {
        float w = t.W[e], m = t.m[e], v = o.kind == DUST_OPT_ADAM ? t.v[e] : 0.f;
        opt_update(o, G[e], w, m, v);
        t.W[e] = w;
        t.m[e] = m;
        if (o.kind == DUST_OPT_ADAM) t.v[e] = v;
        if (t.W_bf16) static_cast<__nv_bfloat16*>(t.W_bf16)[e] = __float2bfloat16_rn(w);
    }
}

}  // namespace

bool make_opt(const dust_opt_params* p, OptParams* o) {
    if (!p || !(p->lr >= 0.f) || !std::isfinite(p->lr) || !(p->weight_decay >= 0.f)) return false;
    *o = OptParams{};
    o->kind = p->kind;
    o->lr = p->lr;
    o->lr_wd = p->lr * p->weight_decay;
    if (p->kind == DUST_OPT_SGD_MOMENTUM) {
        if (!(p->momentum >= 0.f && p->momentum < 1.f)) return false;
        o->mu = p->momentum;
        return true;
    }
    if (p->kind == DUST_OPT_ADAM) {
        if (!(p->beta1 >= 0.f && p->beta1 < 1.f && p->beta2 >= 0.f && p->beta2 < 1.f) ||
            !(p->eps > 0.f) || p->step < 1)
            return false;
        o->b1 = p->beta1;
        o->omb1 = 1.0f - p->beta1;
        o->b2 = p->beta2;
        o->omb2 = 1.0f - p->beta2;
        o->eps = p->eps;
        o->c1 = static_cast<float>(1.0 - std::pow(static_cast<double>(p->beta1), p->step));
        o->c2 = static_cast<float>(1.0 - std::pow(static_cast<double>(p->beta2), p->step));
        return true;
    }
    return false;
}

dust_status opt_launch(const OptParams& o, const float* G, const OptTargets& t, int64_t n,
                       cudaStream_t s) {
    if (n == 0) return DUST_OK;
    const int64_t n4 = std::max<int64_t>(n / 4, 1);
    const unsigned blocks =
        static_cast<unsigned>(std::min<int64_t>((n4 + 255) / 256, static_cast<int64_t>(num_sms()) * 8));
    prof_begin(s);
    opt_step_kernel<<<blocks, 256, 0, s>>>(o, G, t, n);
    prof_end(s, "optimizer_step");
    return cudaGetLastError() == cudaSuccess ? DUST_OK : DUST_ERR_CUDA;
}

}  // namespace dust
