// Centred loss and discounted credit (Dust review page, section "신용 할당": c_s = mean over
// draws of l_s minus l_s; r_t = sum_{s >= t} gamma^(s-t) c_s over later tokens of the same
// sequence).
//
// One block per 128 tokens and a group of up to 128 draw rows.  The block brings its
// [rows, 128] slab of losses into shared memory with bulk asynchronous copies, centres every
// token over the draws, and runs, per draw row, a reverse scan of the affine maps
// r_t = c_t + g_t r_{t+1} (g_t = gamma, or 0 at a segment's last token): each lane composes 4
// consecutive tokens serially and the warp composes the 32 lane maps with shuffles.  Blocks
// are chained from the end of the stream to its start by decoupled look-back: a block
// publishes its aggregate map (A, G), r_first = A + G r_next, then its inclusive value once its
// successor's is known.  Block indices come from an atomic ticket in reverse order, so a block
// only ever waits for blocks that started before it.  Waits are bounded; a wait that runs out
// records the error, writes NaN and still publishes, so no other block waits forever.
// With more than 128 draws, a first kernel computes the per-token mean over all draws and the
// rows are split into groups with independent look-back chains.
#include <algorithm>

#include "dust_device.cuh"
#include "dust_internal.h"

namespace dust {

int g_credit_skip_publish = -1;

namespace {

constexpr int kCB = 128;       // tokens per block
constexpr int kThreads = 128;  // 4 warps; thread j centres token j
constexpr int kRowsMax = 128;  // draw rows per block (row group)
constexpr int kTPL = kCB / 32; // tokens per lane
constexpr int kWarps = kThreads / 32;
constexpr unsigned kAgg = 1u, kInc = 2u;
constexpr int kMaxGroup = 64;

struct CreditLayer {
    const float* loss;
    float* r;
    float* mean;  // [N] per-token mean over all draws (only with several row groups)
    char* state;  // look-back state of row group 0; group g at state + g * state_stride
    int64_t ld_loss, ld_r;
};

// One launch covers the layers and row groups of the table (blockIdx.y = layer * n_groups +
// group); every (layer, group) has its own ticket and look-back state.
template <int kMax>
struct CreditTable {
    CreditLayer layer[kMax];
    const int32_t* cu;
    ErrorWord* ew;
    int64_t N;
    size_t state_stride;
    int n_seq, K, rows, n_groups, nblk, skip_publish, bulk;
    float gamma;
};

size_t state_bytes(int64_t nblk, int rows) {
    return 256 + align_up(static_cast<size_t>(nblk) * kWarps * 4, 256) +
           align_up(static_cast<size_t>(nblk) * rows * 8, 256) +
           align_up(static_cast<size_t>(nblk) * rows * 4, 256);
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(unsigned* p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Bulk asynchronous copy of `bytes` (multiple of 16, 16-byte aligned) global -> shared.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
// Bulk asynchronous copy shared -> global, tracked by the thread's bulk group.
__device__ __forceinline__ void bulk_store(void* dst, const void* smem_src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                     reinterpret_cast<uint64_t>(dst)),
                 "r"(smem_u32(smem_src)), "r"(bytes)
                 : "memory");
}

size_t smem_bytes(int rows) {
    return static_cast<size_t>(rows) * kCB * 4 + static_cast<size_t>(rows) * 4 * 3 + kCB * 4 + 64;
}

// Composes the affine maps of this lane's kTPL tokens (last token first): r_first = A + G r_next.
__device__ __forceinline__ void lane_map(const float4& c, const float4& g, float& A, float& G) {
    A = c.w;
    G = g.w;
    A = fmaf(g.z, A, c.z);
    G = g.z * G;
    A = fmaf(g.y, A, c.y);
    G = g.y * G;
    A = fmaf(g.x, A, c.x);
    G = g.x * G;
}

// Inclusive reverse scan over lanes: lane l ends with the composition of lanes l .. 31.
__device__ __forceinline__ void warp_suffix_scan(int lane, float& A, float& G) {
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float A2 = __shfl_down_sync(0xffffffffu, A, off);
        const float G2 = __shfl_down_sync(0xffffffffu, G, off);
        if (lane + off < 32) {
            A = fmaf(G, A2, A);
            G = G * G2;
        }
    }
}

template <int kMax>
__global__ void __launch_bounds__(kThreads) credit_kernel(const __grid_constant__ CreditTable<kMax> T) {
    const int lyr = blockIdx.y / T.n_groups;
    const int grp = blockIdx.y % T.n_groups;
    const CreditLayer& L = T.layer[lyr];
    char* state = L.state + static_cast<size_t>(grp) * T.state_stride;
    unsigned* ticket = reinterpret_cast<unsigned*>(state);
    unsigned* flags = reinterpret_cast<unsigned*>(state + 256);  // [nblk][kWarps]
    const size_t off_agg = 256 + align_up(static_cast<size_t>(T.nblk) * kWarps * 4, 256);
    float2* agg = reinterpret_cast<float2*>(state + off_agg);
    float* inc = reinterpret_cast<float*>(
        state + off_agg + align_up(static_cast<size_t>(T.nblk) * T.rows * 8, 256));
    const int row0 = grp * T.rows;
    const int R = min(T.rows, T.K - row0);

    extern __shared__ float sm[];
    float* slab = sm;                  // [R][kCB]: loss, then c, then r (16-byte rows)
    float* gval = slab + R * kCB;      // [kCB]: gamma, or 0 at a segment's last token
    float* aggA = gval + kCB;          // [R]
    float* aggG = aggA + R;            // [R]
    float* carry = aggG + R;           // [R]: r at the first token after the block
    uint64_t* bar = reinterpret_cast<uint64_t*>(
        (reinterpret_cast<uintptr_t>(carry + R) + 7) & ~static_cast<uintptr_t>(7));
    __shared__ int s_blk;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        s_blk = T.nblk - 1 - static_cast<int>(atomicAdd(ticket, 1u));
        mbar_init(bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    const int b = s_blk;
    const int64_t t0 = static_cast<int64_t>(b) * kCB;
    const int nb = static_cast<int>(min(static_cast<int64_t>(kCB), T.N - t0));
    const bool bulk = T.bulk && nb == kCB;
    const float* src = L.loss + static_cast<int64_t>(row0) * L.ld_loss + t0;

    if (bulk) {
        if (tid == 0) {
            mbar_arrive_expect_tx(bar, static_cast<uint32_t>(R) * kCB * 4);
            for (int i = 0; i < R; ++i) bulk_load(slab + i * kCB, src + i * L.ld_loss, kCB * 4, bar);
        }
    } else {
        for (int idx = tid; idx < R * kCB; idx += kThreads) {
            const int i = idx / kCB, j = idx % kCB;
            slab[idx] = (j < nb) ? __ldg(src + static_cast<int64_t>(i) * L.ld_loss + j) : 0.f;
        }
    }
    // segment ends (while the copies are in flight)
    gval[tid] = (tid >= nb || t0 + tid == T.N - 1) ? 0.f : T.gamma;
    __syncthreads();
    if (warp == 0) {
        // segment ends e = cu[s] with t0 < e <= t0 + nb end token e - 1 of this block
        int lo = 0, hi = T.n_seq + 1;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (static_cast<int64_t>(__ldg(&T.cu[mid])) > t0) hi = mid;
            else lo = mid + 1;
        }
        for (int s = lo + lane; s <= T.n_seq; s += 32) {
            const int64_t e = __ldg(&T.cu[s]);
            if (e > t0 + nb) break;
            if (e > t0) gval[e - 1 - t0] = 0.f;
        }
    }
    if (bulk) mbar_wait_bounded(bar, 0, T.ew, 301);
    __syncthreads();

    // centring over the draws: mean over all K draws (in this block, or from the mean pass)
    {
        const int j = tid;
        float m;
        if (T.n_groups == 1) {
            m = 0.f;
            for (int i = 0; i < R; ++i) m += slab[i * kCB + j];
            m = m / static_cast<float>(T.K);
        } else {
            m = (j < nb) ? L.mean[t0 + j] : 0.f;
        }
        for (int i = 0; i < R; ++i) slab[i * kCB + j] = m - slab[i * kCB + j];
    }
    __syncthreads();

    // From here each warp owns the rows i = warp + 4 k (one per lane at most) and works on its
    // own: pass 1 (aggregate map per row), look-back with the same warp of the following
    // blocks (its own status flag), pass 2 (the credit).  No block-wide barrier until the store.
    const float4 g4 = *reinterpret_cast<const float4*>(gval + lane * kTPL);
    for (int i = warp; i < R; i += kWarps) {
        const float4 c4 = *reinterpret_cast<const float4*>(slab + i * kCB + lane * kTPL);
        float A, G;
        lane_map(c4, g4, A, G);
        warp_suffix_scan(lane, A, G);
        if (lane == 0) {
            aggA[i] = A;
            aggG[i] = G;
            agg[static_cast<int64_t>(b) * T.rows + i] = make_float2(A, G);
        }
    }
    __syncwarp();

    // Look-back: carry[i] = r at token t0 + kCB of row i.  Only the blocks up to the first one
    // after b that holds a segment end can reach block b (that block's map has G = 0 on every
    // row), so the window of blocks to compose is known from cu_seqlens: their flags are polled
    // in parallel (one lane per block) and their aggregates loaded together; the composition
    // stops early at a block that already published its inclusive value.
    const int my_row = warp + kWarps * lane;  // the row this lane composes
    unsigned* my_flags = flags + warp;        // flag of (block j, this warp) at my_flags[j * kWarps]
    {
        const bool publish = (b != T.skip_publish);
        if (b == T.nblk - 1 || T.gamma == 0.f) {
            if (my_row < R) carry[my_row] = 0.f;
        } else {
            // the aggregates were written by lane 0 itself: its release store publishes them
            if (lane == 0 && publish) st_release(&my_flags[static_cast<int64_t>(b) * kWarps], kAgg);
            int jend;  // the block of the first segment end at or after the first token of b + 1
            {
                const int64_t first = t0 + kCB;
                int lo = 0, hi = T.n_seq + 1;
                while (lo < hi) {
                    const int mid = (lo + hi) >> 1;
                    if (static_cast<int64_t>(__ldg(&T.cu[mid])) > first) hi = mid;
                    else lo = mid + 1;
                }
                const int64_t e = lo <= T.n_seq ? static_cast<int64_t>(__ldg(&T.cu[lo])) : T.N;
                jend = static_cast<int>(min((e - 1) / kCB, static_cast<int64_t>(T.nblk - 1)));
            }
            float accA = 0.f, accG = 1.f;
            const uint64_t start = global_timer_ns();
            bool done = false, failed = false;
            for (int w0 = b + 1; w0 <= jend && !done; w0 += 32) {
                const int j = w0 + lane;
                const bool active = j <= jend;
                unsigned st = 0;
                int timed_out = 0;
                if (active) {
                    st = ld_acquire(&my_flags[static_cast<int64_t>(j) * kWarps]);
                    while (st == 0) {
                        if (global_timer_ns() - start > kWaitLimitNs) {
                            timed_out = 1;
                            break;
                        }
                        __nanosleep(32);
                        st = ld_acquire(&my_flags[static_cast<int64_t>(j) * kWarps]);
                    }
                }
                // each lane acquired its own flag; the warp barrier orders those acquires before
                // every lane's loads of the aggregates below
                __syncwarp();
                if (__any_sync(0xffffffffu, timed_out)) {
                    failed = true;
                    break;
                }
                const unsigned inc_mask = __ballot_sync(0xffffffffu, active && st == kInc);
                const int n_here = min(32, jend - w0 + 1);
                const int stop = inc_mask ? __ffs(inc_mask) - 1 : n_here;  // first INC lane
                if (my_row < R) {
#pragma unroll 8
                    for (int q = 0; q < stop; ++q) {
                        const float2 a = __ldcg(&agg[static_cast<int64_t>(w0 + q) * T.rows + my_row]);
                        accA = fmaf(accG, a.x, accA);
                        accG = accG * a.y;
                    }
                    if (stop < n_here)
                        accA = fmaf(accG, __ldcg(&inc[static_cast<int64_t>(w0 + stop) * T.rows + my_row]),
                                    accA);
                }
                done = stop < n_here || w0 + 31 >= jend;
            }
            if (failed) {
                if (lane == 0) report_error(T.ew, kDevTimeout, b);
                if (my_row < R) carry[my_row] = __int_as_float(0x7fc00000);
            } else if (my_row < R) {
                carry[my_row] = accA;
            }
        }
        if (my_row < R)
            inc[static_cast<int64_t>(b) * T.rows + my_row] = fmaf(aggG[my_row], carry[my_row], aggA[my_row]);
        __syncwarp();
        if (lane == 0 && publish) {
            // the inclusive values were written by every lane: order them before the release
            asm volatile("fence.acq_rel.gpu;" ::: "memory");
            st_release(&my_flags[static_cast<int64_t>(b) * kWarps], kInc);
        }
    }

    // pass 2: this warp's rows again, now with their carries
    for (int i = warp; i < R; i += kWarps) {
        float4 c4 = *reinterpret_cast<const float4*>(slab + i * kCB + lane * kTPL);
        float A, G;
        lane_map(c4, g4, A, G);
        warp_suffix_scan(lane, A, G);
        float eA = __shfl_down_sync(0xffffffffu, A, 1);
        float eG = __shfl_down_sync(0xffffffffu, G, 1);
        if (lane == 31) {
            eA = 0.f;
            eG = 1.f;
        }
        float rn = fmaf(eG, carry[i], eA);
        rn = fmaf(g4.w, rn, c4.w);
        c4.w = rn;
        rn = fmaf(g4.z, rn, c4.z);
        c4.z = rn;
        rn = fmaf(g4.y, rn, c4.y);
        c4.y = rn;
        rn = fmaf(g4.x, rn, c4.x);
        c4.x = rn;
        *reinterpret_cast<float4*>(slab + i * kCB + lane * kTPL) = c4;
    }
    float* dst = L.r + static_cast<int64_t>(row0) * L.ld_r + t0;
    if (bulk) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncthreads();
        if (tid == 0) {
            for (int i = 0; i < R; ++i) bulk_store(dst + i * L.ld_r, slab + i * kCB, kCB * 4);
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        }
    } else {
        __syncthreads();
        for (int idx = tid; idx < R * kCB; idx += kThreads) {
            const int i = idx / kCB, j = idx % kCB;
            if (j < nb) dst[static_cast<int64_t>(i) * L.ld_r + j] = slab[idx];
        }
    }
}

// Per-token mean over all K draws (fixed order), used when the draws span several groups.
template <int kMax>
__global__ void credit_mean_kernel(const __grid_constant__ CreditTable<kMax> T) {
    const CreditLayer& L = T.layer[blockIdx.y];
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < T.N;
         t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float m = 0.f;
        for (int i = 0; i < T.K; ++i) m += __ldg(&L.loss[static_cast<int64_t>(i) * L.ld_loss + t]);
        L.mean[t] = m / static_cast<float>(T.K);
    }
}

int group_rows(int32_t K) { return K <= kRowsMax ? K : kRowsMax; }
int n_groups(int32_t K) { return (K + kRowsMax - 1) / kRowsMax; }

}  // namespace

size_t credit_workspace_bytes(int64_t N, int32_t K) {
    const int64_t nblk = (N + kCB - 1) / kCB;
    const int G = n_groups(K);
    return static_cast<size_t>(G) * state_bytes(nblk, group_rows(K)) +
           (G > 1 ? align_up(static_cast<size_t>(N) * 4, 256) : 0);
}

namespace {

template <int kMax>
void fill_common(CreditTable<kMax>& T, const int32_t* cu, int32_t n_seq, int32_t K, int64_t N,
                 float gamma, int skip, int64_t ld_loss, int64_t ld_r) {
    T.cu = cu;
    T.ew = device_error_word();
    T.N = N;
    T.n_seq = n_seq;
    T.K = K;
    T.rows = group_rows(K);
    T.n_groups = n_groups(K);
    T.nblk = static_cast<int>((N + kCB - 1) / kCB);
    T.state_stride = state_bytes(T.nblk, T.rows);
    T.skip_publish = skip;
    T.gamma = gamma;
    T.bulk = (ld_loss % 4 == 0) && (ld_r % 4 == 0);
}

// Points a layer at its workspace region and clears every group's ticket and flags.
template <int kMax>
bool place_layer(CreditTable<kMax>& T, CreditLayer& L, char* base, cudaStream_t s) {
    L.state = base;
    L.mean = T.n_groups > 1
                 ? reinterpret_cast<float*>(base + static_cast<size_t>(T.n_groups) * T.state_stride)
                 : nullptr;
    for (int g = 0; g < T.n_groups; ++g)
        if (cudaMemsetAsync(base + static_cast<size_t>(g) * T.state_stride, 0,
                            256 + static_cast<size_t>(T.nblk) * kWarps * 4, s) != cudaSuccess)
            return false;
    return true;
}

template <int kMax>
dust_status launch_credit_table(const CreditTable<kMax>& T, int n_layers, cudaStream_t s,
                                const char* name) {
    if (T.n_groups > 1) {
        const unsigned bx = static_cast<unsigned>(
            std::min<int64_t>((T.N + 255) / 256, static_cast<int64_t>(num_sms()) * 8));
        prof_begin(s);
        credit_mean_kernel<kMax><<<dim3(bx, n_layers), 256, 0, s>>>(T);
        prof_end(s, "credit_mean");
    }
    const size_t smem = smem_bytes(T.rows);
    if (cudaFuncSetAttribute(credit_kernel<kMax>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return DUST_ERR_CUDA;
    if (static_cast<int64_t>(n_layers) * T.n_groups > 65535) return DUST_ERR_UNSUPPORTED;
    prof_begin(s);
    credit_kernel<kMax><<<dim3(static_cast<unsigned>(T.nblk), static_cast<unsigned>(n_layers * T.n_groups)),
                          kThreads, smem, s>>>(T);
    prof_end(s, name);
    return cudaGetLastError() == cudaSuccess ? DUST_OK : DUST_ERR_CUDA;
}

}  // namespace

dust_status credit_launch(const float* loss, int64_t ld_loss, int32_t K, int64_t N,
                          const int32_t* cu, int32_t n_seq, float gamma, float* r, int64_t ld_r,
                          void* ws, cudaStream_t s) {
    const int64_t nblk = (N + kCB - 1) / kCB;
    if (nblk > 2147483647LL) return DUST_ERR_UNSUPPORTED;
    CreditTable<1> T;
    fill_common(T, cu, n_seq, K, N, gamma, g_credit_skip_publish, ld_loss, ld_r);
    g_credit_skip_publish = -1;
    T.layer[0].loss = loss;
    T.layer[0].r = r;
    T.layer[0].ld_loss = ld_loss;
    T.layer[0].ld_r = ld_r;
    if (!place_layer(T, T.layer[0], static_cast<char*>(ws), s)) return DUST_ERR_CUDA;
    return launch_credit_table(T, 1, s, "credit_scan");
}

size_t credit_grouped_workspace_bytes(int n_layers, int64_t N, int32_t K) {
    return static_cast<size_t>(n_layers) * credit_workspace_bytes(N, K);
}

dust_status credit_grouped_launch(const CreditLayerArgs* layers, int n, int32_t K, int64_t N,
                                  const int32_t* cu, int32_t n_seq, float gamma, void* ws,
                                  cudaStream_t s) {
    const int64_t nblk = (N + kCB - 1) / kCB;
    if (nblk > 2147483647LL) return DUST_ERR_UNSUPPORTED;
    char* base = static_cast<char*>(ws);
    const size_t per = credit_workspace_bytes(N, K);
    for (int l0 = 0; l0 < n; l0 += kMaxGroup) {
        const int cnt = n - l0 < kMaxGroup ? n - l0 : kMaxGroup;
        CreditTable<kMaxGroup> T;
        bool aligned = true;
        for (int l = 0; l < cnt; ++l)
            aligned = aligned && layers[l0 + l].ld_loss % 4 == 0 && layers[l0 + l].ld_r % 4 == 0;
        fill_common(T, cu, n_seq, K, N, gamma, -1, aligned ? 4 : 1, aligned ? 4 : 1);
        for (int l = 0; l < cnt; ++l) {
            CreditLayer& L = T.layer[l];
            L.loss = layers[l0 + l].loss;
            L.r = layers[l0 + l].r;
            L.ld_loss = layers[l0 + l].ld_loss;
            L.ld_r = layers[l0 + l].ld_r;
            if (!place_layer(T, L, base, s)) return DUST_ERR_CUDA;
            base += per;
        }
        const dust_status st = launch_credit_table(T, cnt, s, "credit_scan_grouped");
        if (st != DUST_OK) return st;
    }
    return DUST_OK;
}

// ------------------------------------------------------------------------------------------
// Credit without a caller workspace.  Some callers cannot allocate device memory at all: a
// plugin run by a host engine that owns every buffer and forbids allocation while it executes,
// or a process working under a fixed memory budget where a cudaMalloc could fail or stall the
// device.  For them the look-back scratch (ticket, status flags, per-block aggregates) lives
// in this fixed device array instead.  Each device that loads the library keeps it until the
// process exits.
// ------------------------------------------------------------------------------------------
constexpr size_t kStaticCreditScratchBytes = 4u << 20;  // 4 MiB per device

static __device__ __align__(256) unsigned char g_credit_scratch[kStaticCreditScratchBytes];

namespace {

// Device address of g_credit_scratch on the current device.  Host code cannot pass the
// array's name to a kernel (on the host it is only a stand-in symbol), so the address is
// looked up once per device, with that device current, and cached.
void* static_credit_scratch() {
    constexpr int kMaxDev = 64;
    static void* addr[kMaxDev] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return nullptr;
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_credit_scratch) != cudaSuccess) return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace

}  // namespace dust

extern "C" dust_status dust_credit_no_alloc(const float* loss, int64_t ld_loss, int32_t K,
                                            int64_t N, const int32_t* cu_seqlens, int32_t n_seq,
                                            float gamma, float* r, int64_t ld_r, void* stream) {
    using namespace dust;
    if (!loss || !r || !cu_seqlens || N < 1 || K < 2 || n_seq < 1 || ld_loss < N || ld_r < N)
        return DUST_ERR_INVALID_ARG;
    if (!(gamma >= 0.f && gamma <= 1.f)) return DUST_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0 ||
        (reinterpret_cast<uintptr_t>(loss) & 15u) != 0 || (reinterpret_cast<uintptr_t>(r) & 15u) != 0)
        return DUST_ERR_INVALID_ARG;
    if (credit_workspace_bytes(N, K) > kStaticCreditScratchBytes) return DUST_ERR_WORKSPACE;
    void* scratch = static_credit_scratch();
    if (!scratch) return DUST_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    CreditTable<1> T;
    fill_common(T, cu_seqlens, n_seq, K, N, gamma, -1, ld_loss, ld_r);
    T.layer[0].loss = loss;
    T.layer[0].r = r;
    T.layer[0].ld_loss = ld_loss;
    T.layer[0].ld_r = ld_r;
    // The tickets and the status flags must start at zero; the array keeps the previous
    // call's contents, so they are cleared on the stream before every launch.
    if (!place_layer(T, T.layer[0], static_cast<char*>(scratch), s)) return DUST_ERR_CUDA;
    return launch_credit_table(T, 1, s, "credit_scan_no_alloc");
}
