// Centred loss and discounted credit (Dust review page, section "신용 할당": c_s = mean over
// draws of l_s minus l_s; r_t = sum_{s >= t} gamma^(s-t) c_s over later tokens of the same
// sequence).
//
// One block per 128 tokens and a group of up to 128 draw rows.  TMA brings the [rows, 128]
// slab of losses into shared memory as four 32-token sub-slabs whose 128-byte lines are
// swizzled (16-byte chunk c of row i sits at chunk c ^ (i mod 8)); the per-token mean over the
// draws is taken by one thread per token.  Then four threads own each draw row, 32 tokens
// each, streamed from the slab in 16-byte chunks: a thread centres its tokens and composes
// their affine maps r_t = c_t + g_t r_{t+1} (g_t = gamma, or 0 at a segment's last token)
// serially, and the four maps of a row are composed with shuffles.  Eight consecutive lanes hold eight different rows
// of the same sub-slab, so every 16-byte shared access of a warp is conflict-free.  Blocks are
// chained from the end of the stream to its start by decoupled look-back: each warp publishes
// its rows' aggregate maps (A, G), r_first = A + G r_next, then their inclusive values once
// the carry from the following blocks is known; a block composes its carry from the
// aggregates of the blocks up to the next segment end (so the result repeats bit for bit) and
// takes an inclusive value only beyond 64 blocks.  Block indices come from an atomic ticket in
// reverse order, so a block only waits for blocks that started before it.  Waits are bounded;
// a wait that runs out records the error, writes NaN and still publishes, so no other block
// waits forever.  The credit is written back into the slab and stored by TMA.  With more than
// 128 draws, a first kernel computes the per-token mean over all draws and the rows are split
// into groups with independent look-back chains.  Leading dimensions that TMA cannot describe
// fall back to plain loads and stores into the same layout.
#include <algorithm>

#include "dust_device.cuh"
#include "dust_internal.h"

namespace dust {

int g_credit_skip_publish = -1;

namespace {

constexpr int kCB = 128;          // tokens per block
constexpr int kSeg = 4;           // threads per draw row
constexpr int kTPT = kCB / kSeg;  // tokens per thread: one 128-byte line
constexpr int kRowsMax = 128;     // draw rows per block (row group)
constexpr int kRowsPerWarp = 32 / kSeg;  // a warp holds kSeg parts of kRowsPerWarp rows
constexpr int kMaxThreads = kRowsMax * kSeg;  // 512
constexpr int kMaxGroup = 64;
// Look-back: blocks read per sweep (one per lane of a row: wider sweeps put more polls on the
// L2 and were slower, 8 blocks by 7% and 16 by 22% on 64 x 4 Mi), and the blocks after b that
// are composed from aggregates alone (64: every segment of up to 8192 tokens).
constexpr int kSweep = 4;
constexpr int kDetBlocks = 64;

struct CreditLayer {
    CUtensorMap tm_loss;  // [K, N] losses, 32 x rows_p boxes, 128-byte swizzle
    CUtensorMap tm_r;     // [K, N] credit, same boxes
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
    int n_seq, K, rows, rows_p, n_groups, nblk, skip_publish, tma;
    int centre;  // 1: centre the losses over the draws first; 0: scan the given reward
    float gamma;
};

int padded_rows(int rows) { return (rows + kRowsPerWarp - 1) / kRowsPerWarp * kRowsPerWarp; }

// Look-back state of one row group: a ticket, then per (block, row) two self-validating 64-bit
// words, so that no fence or separate flag is needed (a naturally aligned 64-bit store is seen
// whole or not at all):
//   aggregate  {A, -G}: published when the sign bit of the high word is set (G >= 0, so -G
//              always has it, -0.0 included); all-zero bits mean "not yet";
//   inclusive  {r_first, 1}: published when the high word is 1.
size_t state_bytes(int64_t nblk, int rows) {
    return 256 + 2 * align_up(static_cast<size_t>(nblk) * rows * 8, 256);
}

size_t smem_bytes(int rows_p) {
    return 1024 + static_cast<size_t>(rows_p) * kCB * 4 + 2 * kCB * 4 +
           static_cast<size_t>(rows_p) * 4 + 16;
}

__device__ __forceinline__ uint64_t ld_relaxed64(const uint64_t* p) {
    uint64_t v;
    asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed64(uint64_t* p, uint64_t v) {
    asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ uint64_t pack2(float lo, uint32_t hi) {
    return static_cast<uint64_t>(__float_as_uint(lo)) | (static_cast<uint64_t>(hi) << 32);
}

// Offset (floats) of (row i, token j) in the slab: sub-slab j / 32 of rows_p 128-byte lines,
// 16-byte chunk (j % 32) / 4 of line i stored at chunk ((j % 32) / 4) ^ (i % 8).
__device__ __forceinline__ int slab_at(int i, int j, int rows_p) {
    return (j >> 5) * rows_p * kTPT + i * kTPT + ((((j & 31) >> 2) ^ (i & 7)) << 2) + (j & 3);
}

// First s in [lo, n_seq] with cu[s] > x (n_seq + 1 if there is none), found by the whole
// warp: each step probes 32 evenly spaced entries of the bracket at once and keeps the part
// that holds the answer, so the dependent loads number log32 of the bracket, not log2.
// cu is non-decreasing and every s < lo has cu[s] <= x.
__device__ __forceinline__ int warp_upper_bound(const int32_t* cu, int n_seq, int64_t x, int lo,
                                                int lane) {
    int hi = n_seq + 1;  // the answer lies in [lo, hi]
    while (lo < hi) {
        const int p = lo + static_cast<int>((static_cast<int64_t>(hi - lo) * lane) >> 5);
        const unsigned m = __ballot_sync(0xffffffffu, static_cast<int64_t>(__ldg(&cu[p])) > x);
        if (m == 0) {
            lo = __shfl_sync(0xffffffffu, p, 31) + 1;
        } else {
            const int k = __ffs(m) - 1;
            const int pk = __shfl_sync(0xffffffffu, p, k);
            const int pprev = __shfl_sync(0xffffffffu, p, k > 0 ? k - 1 : 0);
            lo = k > 0 ? pprev + 1 : lo;
            hi = pk;
        }
    }
    return lo;
}

template <int kMax, int kThr, int kMinBlocks>
__global__ void __launch_bounds__(kThr, kMinBlocks) credit_kernel(const __grid_constant__ CreditTable<kMax> T) {
    const int lyr = blockIdx.y / T.n_groups;
    const int grp = blockIdx.y % T.n_groups;
    const CreditLayer& L = T.layer[lyr];
    char* state = L.state + static_cast<size_t>(grp) * T.state_stride;
    unsigned* ticket = reinterpret_cast<unsigned*>(state);
    uint64_t* aggw = reinterpret_cast<uint64_t*>(state + 256);  // [nblk][rows]
    uint64_t* incw = reinterpret_cast<uint64_t*>(
        state + 256 + align_up(static_cast<size_t>(T.nblk) * T.rows * 8, 256));  // [nblk][rows]
    const int row0 = grp * T.rows;
    const int R = min(T.rows, T.K - row0);
    const int Rp = T.rows_p;

    extern __shared__ uint8_t smem_raw[];
    float* slab = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
    float* gval = slab + Rp * kCB;  // [kCB]: gamma, or 0 at a segment's last token
    float* mean = gval + kCB;       // [kCB]
    float* carry = mean + kCB;      // [Rp]: r at the first token after the block
    uint64_t* bar = reinterpret_cast<uint64_t*>(
        (reinterpret_cast<uintptr_t>(carry + Rp) + 7) & ~static_cast<uintptr_t>(7));
    __shared__ int s_blk, s_jend;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nthr = blockDim.x;
    if (tid == 0) {
        s_blk = T.nblk - 1 - static_cast<int>(atomicAdd(ticket, 1u));
        mbar_init(bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    const int b = s_blk;
    const int64_t t0 = static_cast<int64_t>(b) * kCB;
    const int nb = static_cast<int>(min(static_cast<int64_t>(kCB), T.N - t0));

    if (T.tma) {
        if (tid == 0) {
            mbar_arrive_expect_tx(bar, static_cast<uint32_t>(Rp) * kCB * 4);
#pragma unroll
            for (int sg = 0; sg < kSeg; ++sg)
                tma_load_2d(slab + sg * Rp * kTPT, &L.tm_loss, bar,
                            static_cast<int32_t>(t0) + sg * kTPT, row0);
        }
    } else {
        const float* src = L.loss + static_cast<int64_t>(row0) * L.ld_loss + t0;
        for (int idx = tid; idx < Rp * kCB; idx += nthr) {
            const int i = idx / kCB, j = idx % kCB;
            slab[slab_at(i, j, Rp)] =
                (i < R && j < nb) ? __ldg(src + static_cast<int64_t>(i) * L.ld_loss + j) : 0.f;
        }
    }
    for (int j = tid; j < kCB; j += nthr) gval[j] = (j >= nb || t0 + j == T.N - 1) ? 0.f : T.gamma;
    __syncthreads();
    if (warp == 0) {
        // segment ends e = cu[s] with t0 < e <= t0 + nb end token e - 1 of this block
        const int lo = warp_upper_bound(T.cu, T.n_seq, t0, 0, lane);
        for (int s = lo + lane; s <= T.n_seq; s += 32) {
            const int64_t e = __ldg(&T.cu[s]);
            if (e > t0 + nb) break;
            gval[e - 1 - t0] = 0.f;
        }
        // the block of the first segment end at or after the first token of block b + 1: no
        // look-back reaches past it
        const int hi = warp_upper_bound(T.cu, T.n_seq, t0 + kCB, lo, lane);
        const int64_t e = hi <= T.n_seq ? static_cast<int64_t>(__ldg(&T.cu[hi])) : T.N;
        if (lane == 0)
            s_jend = static_cast<int>(min((e - 1) / kCB, static_cast<int64_t>(T.nblk - 1)));
    }
    if (T.tma) mbar_wait_bounded(bar, 0, T.ew, 301);
    __syncthreads();

    // per-token mean over all K draws (of this block's rows, or from the mean pass)
    if (T.centre) {
        for (int j = tid; j < kCB; j += nthr) {
            float m;
            if (T.n_groups == 1) {
                m = 0.f;
                for (int i = 0; i < R; ++i) m += slab[slab_at(i, j, Rp)];
                m = m / static_cast<float>(T.K);
            } else {
                m = (j < nb) ? L.mean[t0 + j] : 0.f;
            }
            mean[j] = m;
        }
        __syncthreads();
    }

    // Pass 1.  Thread (row i, part sg) owns tokens 32 sg .. 32 sg + 31 of row i and composes
    // their maps from the last token to the first, streaming 16-byte chunks from the slab (the
    // values are not kept in registers, so six CTAs fit on an SM).
    const int i = warp * kRowsPerWarp + lane % kRowsPerWarp;
    const int sg = lane / kRowsPerWarp;
    float* line = slab + sg * Rp * kTPT + i * kTPT;
    // the centred values c = mean - loss of chunk cc of this thread's tokens
    auto centred = [&](int cc) {
        float4 q = *reinterpret_cast<const float4*>(line + ((cc ^ (i & 7)) << 2));
        if (T.centre) {
            const float4 m = *reinterpret_cast<const float4*>(mean + sg * kTPT + 4 * cc);
            q = make_float4(m.x - q.x, m.y - q.y, m.z - q.z, m.w - q.w);
        }
        return q;
    };
    // this thread's map, last token first: r_first = A + G r_next
    float A = 0.f, G = 1.f;
#pragma unroll 2
    for (int c = kTPT / 4 - 1; c >= 0; --c) {
        const float4 g = *reinterpret_cast<const float4*>(gval + sg * kTPT + 4 * c);
        const float4 q = centred(c);
        A = fmaf(g.w, A, q.w);
        G = g.w * G;
        A = fmaf(g.z, A, q.z);
        G = g.z * G;
        A = fmaf(g.y, A, q.y);
        G = g.y * G;
        A = fmaf(g.x, A, q.x);
        G = g.x * G;
    }
    // suffix over the row's four parts (lanes sg, sg + 8, sg + 16, sg + 24 of the warp)
    float sA = A, sG = G;
#pragma unroll
    for (int off = kRowsPerWarp; off < 32; off <<= 1) {
        const float A2 = __shfl_down_sync(0xffffffffu, sA, off);
        const float G2 = __shfl_down_sync(0xffffffffu, sG, off);
        if (lane + off < 32) {
            sA = fmaf(sG, A2, sA);
            sG = sG * G2;
        }
    }
    // the map of the parts after this one (identity for the last part)
    float eA = __shfl_down_sync(0xffffffffu, sA, kRowsPerWarp);
    float eG = __shfl_down_sync(0xffffffffu, sG, kRowsPerWarp);
    if (sg == kSeg - 1) {
        eA = 0.f;
        eG = 1.f;
    }

    // Look-back, per warp and row: only the blocks up to the first one after b that holds a
    // segment end can reach block b (that block's map has G = 0 on every row), so the window
    // b + 1 .. jend is known from cu_seqlens, and the aggregates of the window alone give the
    // carry.  The blocks of the window took their tickets just before b, so their inclusive
    // values are rarely out yet: up to kDetBlocks blocks after b are read as aggregates only, in
    // sweeps of kSweep blocks, lane (row r, part q) polling blocks base + q + 4k (k < kSweep / 4),
    // and the four lanes of a row compose the answers in block order.  The carry is then the
    // same fixed-order composition in every run, and the credit repeats bit for bit.  A window
    // longer than kDetBlocks (a segment of more than 8192 tokens) is walked on four blocks at a
    // time, each polled for its inclusive value first, stopping at the first one found; its
    // last bits then depend on which blocks had published.
    const bool row_ok = i < R;
    {
        const bool publish = (b != T.skip_publish);
        float carry_i = 0.f;
        // every block publishes its aggregate (the last one too: the aggregate-only sweep of
        // the blocks before it reads it)
        if (T.gamma != 0.f && sg == 0 && row_ok && publish)
            st_relaxed64(&aggw[static_cast<int64_t>(b) * T.rows + i],
                         pack2(sA, __float_as_uint(-sG)));
        if (b != T.nblk - 1 && T.gamma != 0.f) {
            const int jend = s_jend;
            float accA = 0.f, accG = 1.f;
            bool done = !row_ok, failed = false;
            const uint64_t start = global_timer_ns();
            // sweeps of kSweep blocks read as aggregates only, up to kDetBlocks after b
            const int det_end = min(jend, b + kDetBlocks);
            int base = b + 1;
            for (; base <= det_end && !__all_sync(0xffffffffu, done); base += kSweep) {
                constexpr int kPer = kSweep / kSeg;  // blocks per lane
                float va[kPer], vg[kPer];
                bool pend[kPer];
                int kind = 0;  // 0: answered; 3: a wait ran out
#pragma unroll
                for (int k = 0; k < kPer; ++k) {
                    va[k] = 0.f;
                    vg[k] = 1.f;
                    pend[k] = !done && base + sg + kSeg * k <= det_end;
                }
                while (true) {
                    uint64_t w[kPer];
#pragma unroll
                    for (int k = 0; k < kPer; ++k)
                        if (pend[k])
                            w[k] = ld_relaxed64(
                                &aggw[static_cast<int64_t>(base + sg + kSeg * k) * T.rows + i]);
                    bool any = false;
#pragma unroll
                    for (int k = 0; k < kPer; ++k) {
                        if (pend[k] && (static_cast<uint32_t>(w[k] >> 32) & 0x80000000u)) {
                            va[k] = __uint_as_float(static_cast<uint32_t>(w[k]));
                            vg[k] = -__uint_as_float(static_cast<uint32_t>(w[k] >> 32));
                            pend[k] = false;
                        }
                        any = any || pend[k];
                    }
                    if (!any) break;
                    if (global_timer_ns() - start > kWaitLimitNs) {
                        kind = 3;
                        break;
                    }
                    __nanosleep(32);
                }
                // compose blocks base .. base + kSweep - 1 in order: block base + q + 4k is lane
                // (r, q)'s slot k; blocks past det_end carry the identity map
#pragma unroll
                for (int k = 0; k < kPer; ++k) {
#pragma unroll
                    for (int q = 0; q < kSeg; ++q) {
                        const int src = lane % kRowsPerWarp + kRowsPerWarp * q;
                        const float aq = __shfl_sync(0xffffffffu, va[k], src);
                        const float gq = __shfl_sync(0xffffffffu, vg[k], src);
                        if (!done) {
                            accA = fmaf(accG, aq, accA);
                            accG = accG * gq;
                        }
                    }
                }
                int kq = kind;  // the row's: any of its four lanes ran out
#pragma unroll
                for (int q = 0; q < kSeg; ++q)
                    kq = max(kq, __shfl_sync(0xffffffffu, kind,
                                             lane % kRowsPerWarp + kRowsPerWarp * q));
                if (kq == 3 && !done) {
                    failed = true;
                    done = true;
                }
            }
            if (det_end == jend) done = true;  // the window was composed from aggregates alone
            base = det_end + 1;
            for (; base <= jend && !__all_sync(0xffffffffu, done); base += kSeg) {
                const int j = base + sg;
                int kind = 0;  // 1: aggregate (va, vg); 2: inclusive value va; 3: wait ran out
                float va = 0.f, vg = 1.f;
                if (!done && j <= jend) {
                    const int64_t at = static_cast<int64_t>(j) * T.rows + i;
                    while (true) {
                        const uint64_t wi = ld_relaxed64(&incw[at]);
                        if (static_cast<uint32_t>(wi >> 32) == 1u) {
                            kind = 2;
                            va = __uint_as_float(static_cast<uint32_t>(wi));
                            break;
                        }
                        const uint64_t wa = ld_relaxed64(&aggw[at]);
                        if (static_cast<uint32_t>(wa >> 32) & 0x80000000u) {
                            kind = 1;
                            va = __uint_as_float(static_cast<uint32_t>(wa));
                            vg = -__uint_as_float(static_cast<uint32_t>(wa >> 32));
                            break;
                        }
                        if (global_timer_ns() - start > kWaitLimitNs) {
                            kind = 3;
                            break;
                        }
                        __nanosleep(32);
                    }
                }
#pragma unroll
                for (int q = 0; q < kSeg; ++q) {
                    const int src = lane % kRowsPerWarp + kRowsPerWarp * q;
                    const int kq = __shfl_sync(0xffffffffu, kind, src);
                    const float aq = __shfl_sync(0xffffffffu, va, src);
                    const float gq = __shfl_sync(0xffffffffu, vg, src);
                    if (!done) {
                        if (kq == 3) {
                            failed = true;
                            done = true;
                        } else if (kq == 2) {
                            accA = fmaf(accG, aq, accA);
                            done = true;
                        } else if (kq == 1) {
                            accA = fmaf(accG, aq, accA);
                            accG = accG * gq;
                        }
                    }
                }
            }
            if (failed) {
                if (sg == 0) report_error(T.ew, kDevTimeout, b);
                carry_i = __int_as_float(0x7fc00000);
            } else {
                carry_i = accA;
            }
        }
        if (sg == 0) {
            carry[i] = carry_i;
            if (row_ok && publish)
                st_relaxed64(&incw[static_cast<int64_t>(b) * T.rows + i],
                             pack2(fmaf(sG, carry_i, sA), 1u));
        }
        __syncwarp();
    }

    // Pass 2: the credit of this thread's tokens, from the carry of its row, back into the slab
    // (the centred values are formed again from the slab, in the same arithmetic).
    {
        float rn = fmaf(eG, carry[i], eA);
#pragma unroll 2
        for (int c = kTPT / 4 - 1; c >= 0; --c) {
            const float4 g = *reinterpret_cast<const float4*>(gval + sg * kTPT + 4 * c);
            const float4 cv = centred(c);
            float4 q;
            rn = fmaf(g.w, rn, cv.w);
            q.w = rn;
            rn = fmaf(g.z, rn, cv.z);
            q.z = rn;
            rn = fmaf(g.y, rn, cv.y);
            q.y = rn;
            rn = fmaf(g.x, rn, cv.x);
            q.x = rn;
            *reinterpret_cast<float4*>(line + ((c ^ (i & 7)) << 2)) = q;
        }
    }
    if (T.tma) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncthreads();
        if (tid == 0) {
#pragma unroll
            for (int q = 0; q < kSeg; ++q)
                tma_store_2d(&L.tm_r, slab + q * Rp * kTPT, static_cast<int32_t>(t0) + q * kTPT,
                             row0);
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        }
    } else {
        __syncthreads();
        float* dst = L.r + static_cast<int64_t>(row0) * L.ld_r + t0;
        for (int idx = tid; idx < R * kCB; idx += nthr) {
            const int ii = idx / kCB, j = idx % kCB;
            if (j < nb) dst[static_cast<int64_t>(ii) * L.ld_r + j] = slab[slab_at(ii, j, Rp)];
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
                 float gamma, int skip, int64_t ld_loss, int64_t ld_r, int centre = 1) {
    T.cu = cu;
    T.centre = centre;
    T.ew = device_error_word();
    T.N = N;
    T.n_seq = n_seq;
    T.K = K;
    T.rows = group_rows(K);
    T.rows_p = padded_rows(T.rows);
    T.n_groups = n_groups(K);
    T.nblk = static_cast<int>((N + kCB - 1) / kCB);
    T.state_stride = state_bytes(T.nblk, T.rows);
    T.skip_publish = skip;
    T.gamma = gamma;
    T.tma = (ld_loss % 4 == 0) && (ld_r % 4 == 0);
}

// Points a layer at its workspace region, clears every group's ticket and look-back words (unless
// the caller clears the regions of several layers at once), and encodes its TMA descriptors (a
// table whose descriptors cannot all be encoded uses plain loads).
template <int kMax>
bool place_layer(CreditTable<kMax>& T, CreditLayer& L, char* base, cudaStream_t s,
                 bool clear = true) {
    L.state = base;
    if (T.tma &&
        !(make_tmap_f32_2d_sw128(&L.tm_loss, L.loss, static_cast<uint64_t>(T.K),
                                 static_cast<uint64_t>(T.N), static_cast<uint64_t>(L.ld_loss),
                                 static_cast<uint32_t>(T.rows_p)) &&
          make_tmap_f32_2d_sw128(&L.tm_r, L.r, static_cast<uint64_t>(T.K),
                                 static_cast<uint64_t>(T.N), static_cast<uint64_t>(L.ld_r),
                                 static_cast<uint32_t>(T.rows_p))))
        T.tma = 0;
    L.mean = T.n_groups > 1 && T.centre
                 ? reinterpret_cast<float*>(base + static_cast<size_t>(T.n_groups) * T.state_stride)
                 : nullptr;
    // the groups' states are contiguous
    return !clear || cudaMemsetAsync(base, 0, static_cast<size_t>(T.n_groups) * T.state_stride,
                                     s) == cudaSuccess;
}

template <int kMax>
dust_status launch_credit_table(const CreditTable<kMax>& T, int n_layers, cudaStream_t s,
                                const char* name) {
    if (T.n_groups > 1 && T.centre) {
        const unsigned bx = static_cast<unsigned>(
            std::min<int64_t>((T.N + 255) / 256, static_cast<int64_t>(num_sms()) * 8));
        prof_begin(s);
        credit_mean_kernel<kMax><<<dim3(bx, n_layers), 256, 0, s>>>(T);
        prof_end(s, "credit_mean");
    }
    const size_t smem = smem_bytes(T.rows_p);
    const int threads = kSeg * T.rows_p;
    // up to 64 rows (256 threads): six resident blocks (42 registers each); 128 rows: two
    auto kern = threads <= 256 ? credit_kernel<kMax, 256, 6> : credit_kernel<kMax, kMaxThreads, 2>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return DUST_ERR_CUDA;
    if (static_cast<int64_t>(n_layers) * T.n_groups > 65535) return DUST_ERR_UNSUPPORTED;
    prof_begin(s);
    kern<<<dim3(static_cast<unsigned>(T.nblk), static_cast<unsigned>(n_layers * T.n_groups)),
           threads, smem, s>>>(T);
    prof_end(s, name);
    return cudaGetLastError() == cudaSuccess ? DUST_OK : DUST_ERR_CUDA;
}

}  // namespace

dust_status credit_launch(const float* loss, int64_t ld_loss, int32_t K, int64_t N,
                          const int32_t* cu, int32_t n_seq, float gamma, float* r, int64_t ld_r,
                          void* ws, cudaStream_t s, int centre) {
    const int64_t nblk = (N + kCB - 1) / kCB;
    if (nblk > 2147483647LL) return DUST_ERR_UNSUPPORTED;
    CreditTable<1> T;
    fill_common(T, cu, n_seq, K, N, gamma, g_credit_skip_publish, ld_loss, ld_r, centre);
    g_credit_skip_publish = -1;
    T.layer[0].loss = loss;
    T.layer[0].r = r;
    T.layer[0].ld_loss = ld_loss;
    T.layer[0].ld_r = ld_r;
    if (!place_layer(T, T.layer[0], static_cast<char*>(ws), s)) return DUST_ERR_CUDA;
    return launch_credit_table(T, 1, s, centre ? "credit_scan" : "discounted_credit_scan");
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
        // the table's layers' regions are contiguous: one memset clears their states (and the
        // per-token means, which the mean pass rewrites)
        if (cudaMemsetAsync(base, 0, static_cast<size_t>(cnt) * per, s) != cudaSuccess)
            return DUST_ERR_CUDA;
        for (int l = 0; l < cnt; ++l) {
            CreditLayer& L = T.layer[l];
            L.loss = layers[l0 + l].loss;
            L.r = layers[l0 + l].r;
            L.ld_loss = layers[l0 + l].ld_loss;
            L.ld_r = layers[l0 + l].ld_r;
            if (!place_layer(T, L, base, s, false)) return DUST_ERR_CUDA;
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
// device.  For them the look-back scratch (ticket and per-block look-back words) lives
// in this fixed device array instead.  Each device that loads the library keeps it until the
// process exits.
// ------------------------------------------------------------------------------------------
constexpr size_t kStaticCreditScratchBytes = 4u << 20;  // 4 MiB per device

static __device__ __align__(256) unsigned char g_credit_scratch[kStaticCreditScratchBytes];

namespace {

// Device address of g_credit_scratch on the current device.  Host code cannot pass the
// array's name to a kernel (on the host it is only a stand-in symbol), so the address is
// looked up with cudaGetSymbolAddress once per device, with that device current, and cached
// (thread-safe; looked up again if the device's context was reset).
void* static_credit_scratch() {
    static SymbolAddressCache cache;
    return cache.get([] {
        void* p = nullptr;
        return cudaGetSymbolAddress(&p, g_credit_scratch) == cudaSuccess ? p : nullptr;
    });
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
    // The tickets and the look-back words must start at zero; the array keeps the previous
    // call's contents, so they are cleared on the stream before every launch.
    if (!place_layer(T, T.layer[0], static_cast<char*>(scratch), s)) return DUST_ERR_CUDA;
    return launch_credit_table(T, 1, s, "credit_scan_no_alloc");
}
