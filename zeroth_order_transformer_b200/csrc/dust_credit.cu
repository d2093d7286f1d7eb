// Centred loss and discounted credit (Dust review page, section "신용 할당": c_s = mean over
// draws of l_s minus l_s; r_t = sum_{s >= t} gamma^(s-t) c_s over later tokens of the same
// sequence).
//
// One block per 256 tokens and all K draws.  The block stages its [K, 256] slab of losses in
// shared memory, centres every token over the draws, and runs, per draw row, a reverse scan
// of the affine maps r_t = c_t + g_t r_{t+1} (g_t = gamma, or 0 at a segment's last token):
// each lane composes 8 consecutive tokens serially, the warp composes the 32 lane maps with
// shuffles.  Blocks are chained from the end of the stream to its start by decoupled
// look-back: a block publishes its aggregate map (A, G) with r_first = A + G * r_next, then
// its inclusive value once its successor's is known.  Block indices come from an atomic
// ticket in reverse order, so a block only ever waits for blocks that started before it.
// Waits are bounded; a wait that runs out records the error, writes NaN and still publishes,
// so no other block waits forever.
#include "dust_device.cuh"
#include "dust_internal.h"

namespace dust {

int g_credit_skip_publish = -1;

namespace {

constexpr int kCB = 256;       // tokens per block
constexpr int kThreads = 256;  // 8 warps
constexpr int kKMax = 128;     // draws held in shared memory at once
constexpr unsigned kAgg = 1u, kInc = 2u;

struct CreditLayer {
    const float* loss;
    float* r;
    unsigned* ticket;
    unsigned* flags;  // [nblk]
    float2* agg;      // [nblk, K]
    float* inc;       // [nblk, K]
    int64_t ld_loss, ld_r;
};

// One launch covers the layers of the table (blockIdx.y = layer); every layer has its own
// ticket and look-back state, so blocks of different layers never wait for one another.
template <int kMax>
struct CreditTable {
    CreditLayer layer[kMax];
    const int32_t* cu;
    ErrorWord* ew;
    int64_t N;
    int n_seq, K, nblk, skip_publish;
    float gamma;
};

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(unsigned* p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

size_t smem_bytes(int K) {
    return static_cast<size_t>(K) * kCB * 4 + kCB * 4 + static_cast<size_t>(K) * 32 * 4 * 2 +
           static_cast<size_t>(K) * 4 * 3 + kCB;
}

template <int kMax>
__global__ void __launch_bounds__(kThreads) credit_kernel(const __grid_constant__ CreditTable<kMax> T) {
    const CreditLayer& L = T.layer[blockIdx.y];
    extern __shared__ float sm[];
    const int K = T.K;
    float* slab = sm;                 // [K][kCB]: loss, then c, then r
    float* exA = slab + K * kCB;      // [K][32]: map of the tokens after each lane's range
    float* exG = exA + K * 32;
    float* carry = exG + K * 32;      // [K]: r at the first token after the block
    float* aggA = carry + K;          // [K]
    float* aggG = aggA + K;           // [K]
    float* mean = aggG + K;           // [kCB]
    unsigned char* isend = reinterpret_cast<unsigned char*>(mean + kCB);  // [kCB]
    __shared__ int s_blk;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) s_blk = T.nblk - 1 - static_cast<int>(atomicAdd(L.ticket, 1u));
    __syncthreads();
    const int b = s_blk;
    const int64_t t0 = static_cast<int64_t>(b) * kCB;
    const int nb = static_cast<int>(min(static_cast<int64_t>(kCB), T.N - t0));

    for (int idx = tid; idx < K * kCB; idx += kThreads) {
        const int i = idx / kCB, j = idx % kCB;
        slab[idx] = (j < nb) ? __ldg(&L.loss[static_cast<int64_t>(i) * L.ld_loss + t0 + j]) : 0.f;
    }
    for (int j = tid; j < kCB; j += kThreads) isend[j] = (j >= nb || t0 + j == T.N - 1) ? 1 : 0;
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
            if (e > t0) isend[e - 1 - t0] = 1;
        }
    }
    // centring over the draws (the mean includes every draw)
    for (int j = tid; j < kCB; j += kThreads) {
        float m = 0.f;
        for (int i = 0; i < K; ++i) m += slab[i * kCB + j];
        m = m / static_cast<float>(K);
        for (int i = 0; i < K; ++i) slab[i * kCB + j] = m - slab[i * kCB + j];
    }
    __syncthreads();

    const float gam = T.gamma;
    for (int i = warp; i < K; i += kThreads / 32) {
        const float* row = slab + i * kCB + lane * 8;
        float A = 0.f, G = 1.f;
#pragma unroll
        for (int k = 7; k >= 0; --k) {
            const float g = isend[lane * 8 + k] ? 0.f : gam;
            A = row[k] + g * A;
            G = g * G;
        }
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float A2 = __shfl_down_sync(0xffffffffu, A, off);
            const float G2 = __shfl_down_sync(0xffffffffu, G, off);
            if (lane + off < 32) {
                A = A + G * A2;
                G = G * G2;
            }
        }
        float eA = __shfl_down_sync(0xffffffffu, A, 1);
        float eG = __shfl_down_sync(0xffffffffu, G, 1);
        if (lane == 31) {
            eA = 0.f;
            eG = 1.f;
        }
        exA[i * 32 + lane] = eA;
        exG[i * 32 + lane] = eG;
        if (lane == 0) {
            aggA[i] = A;
            aggG[i] = G;
            L.agg[static_cast<int64_t>(b) * K + i] = make_float2(A, G);
        }
    }
    __syncthreads();

    if (warp == 0) {
        const bool publish = (b != T.skip_publish);
        if (b == T.nblk - 1) {
            for (int i = lane; i < K; i += 32) carry[i] = 0.f;
        } else {
            if (lane == 0) {
                __threadfence();
                if (publish) st_release(&L.flags[b], kAgg);
            }
            __syncwarp();
            constexpr int kRows = kKMax / 32;
            float accA[kRows], accG[kRows];
#pragma unroll
            for (int k = 0; k < kRows; ++k) {
                accA[k] = 0.f;
                accG[k] = 1.f;
            }
            int j = b + 1;
            const uint64_t start = global_timer_ns();
            while (true) {
                if (j >= T.nblk) {
#pragma unroll
                    for (int k = 0; k < kRows; ++k)
                        if (lane + 32 * k < K) carry[lane + 32 * k] = accA[k];
                    break;
                }
                unsigned st = 0;
                int timed_out = 0;
                if (lane == 0) {
                    st = ld_acquire(&L.flags[j]);
                    while (st == 0) {
                        if (global_timer_ns() - start > kWaitLimitNs) {
                            timed_out = 1;
                            break;
                        }
                        __nanosleep(64);
                        st = ld_acquire(&L.flags[j]);
                    }
                }
                st = __shfl_sync(0xffffffffu, st, 0);
                timed_out = __shfl_sync(0xffffffffu, timed_out, 0);
                __threadfence();
                if (timed_out) {
                    if (lane == 0) report_error(T.ew, kDevTimeout, b);
                    for (int i = lane; i < K; i += 32) carry[i] = __int_as_float(0x7fc00000);
                    break;
                }
                if (st == kInc) {
#pragma unroll
                    for (int k = 0; k < kRows; ++k) {
                        const int i = lane + 32 * k;
                        if (i < K)
                            carry[i] = accA[k] + accG[k] * __ldcg(&L.inc[static_cast<int64_t>(j) * K + i]);
                    }
                    break;
                }
                bool all_zero = true;
#pragma unroll
                for (int k = 0; k < kRows; ++k) {
                    const int i = lane + 32 * k;
                    if (i < K) {
                        const float2 a = __ldcg(&L.agg[static_cast<int64_t>(j) * K + i]);
                        accA[k] = accA[k] + accG[k] * a.x;
                        accG[k] = accG[k] * a.y;
                        all_zero = all_zero && (accG[k] == 0.f);
                    }
                }
                if (__all_sync(0xffffffffu, all_zero)) {
#pragma unroll
                    for (int k = 0; k < kRows; ++k)
                        if (lane + 32 * k < K) carry[lane + 32 * k] = accA[k];
                    break;
                }
                ++j;
            }
        }
        for (int i = lane; i < K; i += 32)
            L.inc[static_cast<int64_t>(b) * K + i] = aggA[i] + aggG[i] * carry[i];
        __syncwarp();
        if (lane == 0) {
            __threadfence();
            if (publish) st_release(&L.flags[b], kInc);
        }
    }
    __syncthreads();

    for (int i = warp; i < K; i += kThreads / 32) {
        float* row = slab + i * kCB + lane * 8;
        float rn = exA[i * 32 + lane] + exG[i * 32 + lane] * carry[i];
#pragma unroll
        for (int k = 7; k >= 0; --k) {
            const float g = isend[lane * 8 + k] ? 0.f : gam;
            rn = row[k] + g * rn;
            row[k] = rn;
        }
    }
    __syncthreads();
    for (int idx = tid; idx < K * kCB; idx += kThreads) {
        const int i = idx / kCB, j = idx % kCB;
        if (j < nb) L.r[static_cast<int64_t>(i) * L.ld_r + t0 + j] = slab[idx];
    }
}

}  // namespace

size_t credit_workspace_bytes(int64_t N, int32_t K) {
    const int64_t nblk = (N + kCB - 1) / kCB;
    return 256 + align_up(static_cast<size_t>(nblk) * 4, 256) +
           align_up(static_cast<size_t>(nblk) * K * 8, 256) +
           align_up(static_cast<size_t>(nblk) * K * 4, 256);
}

namespace {

// Points a layer's look-back state at `base` (credit_workspace_bytes(N, K) bytes) and clears
// the ticket and flags on the stream.
bool place_credit_state(CreditLayer& L, char* base, int64_t nblk, int32_t K, cudaStream_t s) {
    L.ticket = reinterpret_cast<unsigned*>(base);
    L.flags = reinterpret_cast<unsigned*>(base + 256);
    const size_t off_agg = 256 + align_up(static_cast<size_t>(nblk) * 4, 256);
    L.agg = reinterpret_cast<float2*>(base + off_agg);
    L.inc = reinterpret_cast<float*>(base + off_agg + align_up(static_cast<size_t>(nblk) * K * 8, 256));
    return cudaMemsetAsync(base, 0, 256 + static_cast<size_t>(nblk) * 4, s) == cudaSuccess;
}

template <int kMax>
dust_status launch_credit_table(const CreditTable<kMax>& T, int n_layers, cudaStream_t s,
                                const char* name) {
    const size_t smem = smem_bytes(T.K);
    if (cudaFuncSetAttribute(credit_kernel<kMax>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return DUST_ERR_CUDA;
    prof_begin(s);
    credit_kernel<kMax><<<dim3(static_cast<unsigned>(T.nblk), static_cast<unsigned>(n_layers)),
                          kThreads, smem, s>>>(T);
    prof_end(s, name);
    return cudaGetLastError() == cudaSuccess ? DUST_OK : DUST_ERR_CUDA;
}

template <int kMax>
void fill_common(CreditTable<kMax>& T, const int32_t* cu, int32_t n_seq, int32_t K, int64_t N,
                 float gamma, int skip) {
    T.cu = cu;
    T.ew = device_error_word();
    T.N = N;
    T.n_seq = n_seq;
    T.K = K;
    T.nblk = static_cast<int>((N + kCB - 1) / kCB);
    T.skip_publish = skip;
    T.gamma = gamma;
}

constexpr int kMaxGroup = 64;

}  // namespace

dust_status credit_launch(const float* loss, int64_t ld_loss, int32_t K, int64_t N,
                          const int32_t* cu, int32_t n_seq, float gamma, float* r, int64_t ld_r,
                          void* ws, cudaStream_t s) {
    if (K > kKMax) return DUST_ERR_UNSUPPORTED;
    const int64_t nblk = (N + kCB - 1) / kCB;
    if (nblk > 2147483647LL) return DUST_ERR_UNSUPPORTED;
    CreditTable<1> T;
    fill_common(T, cu, n_seq, K, N, gamma, g_credit_skip_publish);
    g_credit_skip_publish = -1;
    T.layer[0].loss = loss;
    T.layer[0].r = r;
    T.layer[0].ld_loss = ld_loss;
    T.layer[0].ld_r = ld_r;
    if (!place_credit_state(T.layer[0], static_cast<char*>(ws), nblk, K, s)) return DUST_ERR_CUDA;
    return launch_credit_table(T, 1, s, "credit_scan");
}

size_t credit_grouped_workspace_bytes(int n_layers, int64_t N, int32_t K) {
    return static_cast<size_t>(n_layers) * credit_workspace_bytes(N, K);
}

dust_status credit_grouped_launch(const CreditLayerArgs* layers, int n, int32_t K, int64_t N,
                                  const int32_t* cu, int32_t n_seq, float gamma, void* ws,
                                  cudaStream_t s) {
    if (K > kKMax) return DUST_ERR_UNSUPPORTED;
    const int64_t nblk = (N + kCB - 1) / kCB;
    if (nblk > 2147483647LL) return DUST_ERR_UNSUPPORTED;
    char* base = static_cast<char*>(ws);
    const size_t per = credit_workspace_bytes(N, K);
    for (int l0 = 0; l0 < n; l0 += kMaxGroup) {
        const int cnt = n - l0 < kMaxGroup ? n - l0 : kMaxGroup;
        CreditTable<kMaxGroup> T;
        fill_common(T, cu, n_seq, K, N, gamma, -1);
        for (int l = 0; l < cnt; ++l) {
            CreditLayer& L = T.layer[l];
            L.loss = layers[l0 + l].loss;
            L.r = layers[l0 + l].r;
            L.ld_loss = layers[l0 + l].ld_loss;
            L.ld_r = layers[l0 + l].ld_r;
            if (!place_credit_state(L, base, nblk, K, s)) return DUST_ERR_CUDA;
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
    if (K > kKMax) return DUST_ERR_UNSUPPORTED;
    if (credit_workspace_bytes(N, K) > kStaticCreditScratchBytes) return DUST_ERR_WORKSPACE;
    void* scratch = static_credit_scratch();
    if (!scratch) return DUST_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t nblk = (N + kCB - 1) / kCB;
    CreditTable<1> T;
    fill_common(T, cu_seqlens, n_seq, K, N, gamma, -1);
    T.layer[0].loss = loss;
    T.layer[0].r = r;
    T.layer[0].ld_loss = ld_loss;
    T.layer[0].ld_r = ld_r;
    // The ticket and the status flags must start at zero; the array keeps the previous
    // call's contents, so they are cleared on the stream before every launch.
    if (!place_credit_state(T.layer[0], static_cast<char*>(scratch), nblk, K, s))
        return DUST_ERR_CUDA;
    return launch_credit_table(T, 1, s, "credit_scan_no_alloc");
}
