/*
 * Dust estimator oracle: plain, slow, fp64 CPU reference of the token-level
 * node-perturbation gradient estimator for one linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call
 * this file: only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark use it.  It shares no code with the CUDA kernels.
 *
 * Source of every formula: the Dust review page (koala.ai.kr, "Dust: 역전파 없이
 * 트랜스포머를 사전학습하다"), section "신용 할당(credit assignment): 보상에서
 * 기울기까지":
 *   noise equation          y_t -> y_t + sigma a_t,  a_t ~ N(0, I), independent per token
 *   centred loss            c_s = mean-over-draws(l_s) - l_s
 *   credit equation         r_t = sum_{s >= t} gamma^(s-t) c_s  (later tokens of the sequence)
 *   output-error equation   g_t = -(1/(K sigma)) sum_i r_t^(i) a_t^(i)
 *   weight-estimate eq.     G_W = sum_t g_t x_t^T
 * and, for the "next" rows: the optimizer steps on G_W (section "설정", section "Adam에서도
 * 통할까?"), the LM-head cross-entropy on cached logits and the attention-internal reward
 * c_s = -<ghat_s, delta_o_s> (section "간섭(interference) 줄이기").
 * The page fixes no random generator.  The one used here is Philox4x32-10
 * (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3",
 * SC'11), written from that paper's description, with the Box-Muller transform
 * (Box & Muller 1958) on uniforms u(w) = (2*(w >> 9) + 1) * 2^-24.
 * Counter of the quad that holds channel o of token t in draw i of layer L:
 *   (o >> 2, token_offset + t, draw_offset + i, L), key = (seed lo32, seed hi32);
 * channel o takes normal z[o & 3] of that quad.
 *
 * Every loop below is the plain definition; OpenMP only splits independent
 * outer loops (tokens or output rows) across threads and never changes the
 * order in which one output element is summed.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_get_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Philox4x32 with 10 rounds (Salmon et al. 2011, section 3 "Philox"): each round
 * multiplies words 0 and 2 by the two round multipliers into 64-bit products,
 * and the new block is (hi(M1*c2) ^ c1 ^ k0, lo(M1*c2), hi(M0*c0) ^ c3 ^ k1,
 * lo(M0*c0)); the key is bumped by the two Weyl constants between rounds. */
void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += PHILOX_W0;
            k1 += PHILOX_W1;
        }
        uint64_t p0 = (uint64_t)PHILOX_M0 * (uint64_t)c0;
        uint64_t p1 = (uint64_t)PHILOX_M1 * (uint64_t)c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        uint32_t n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* u(w) = (2 * (w >> 9) + 1) * 2^-24: the top 23 bits, centred in their cell; never 0 or 1. */
double oracle_uniform(uint32_t w)
{
    return ldexp(2.0 * (double)(w >> 9) + 1.0, -24);
}

/* Box-Muller on the four words of one Philox block: (w0, w1) -> (z0, z1), (w2, w3) -> (z2, z3). */
void oracle_box_muller4(const uint32_t w[4], double z[4])
{
    const double two_pi = 6.283185307179586476925286766559;
    for (int p = 0; p < 2; ++p) {
        double rho = sqrt(-2.0 * log(oracle_uniform(w[2 * p])));
        double theta = two_pi * oracle_uniform(w[2 * p + 1]);
        z[2 * p] = rho * cos(theta);
        z[2 * p + 1] = rho * sin(theta);
    }
}

/* The four normals a[4q .. 4q+3] of token t (global), draw i (global), layer L. */
void oracle_normal_quad(uint64_t seed, uint32_t q, uint32_t t, uint32_t i, uint32_t layer,
                        double z[4])
{
    uint32_t ctr[4] = {q, t, i, layer};
    uint32_t key[2] = {(uint32_t)(seed & 0xffffffffu), (uint32_t)(seed >> 32)};
    uint32_t w[4];
    oracle_philox4x32_10(ctr, key, w);
    oracle_box_muller4(w, z);
}

/* Streaming statistics of the generator's normals, for the distribution pins at sizes whose
 * samples would not fit in memory: blocks j = 0 .. n_blocks-1 with counter
 * (j mod 1024, j / 1024, draw, layer) give 4 n_blocks normals.  sums[0] = sum z, sums[1] =
 * sum z^2; hist[0] counts z < lo, hist[1 + b] counts z in bin b of n_bins equal bins of
 * [lo, hi), hist[n_bins + 1] counts z >= hi. */
void oracle_normal_stats(uint64_t seed, uint32_t draw, uint32_t layer, int64_t n_blocks,
                         int32_t n_bins, double lo, double hi, double* sums, int64_t* hist)
{
    const double scale = (double)n_bins / (hi - lo);
    sums[0] = 0.0;
    sums[1] = 0.0;
    memset(hist, 0, sizeof(int64_t) * (size_t)(n_bins + 2));
#pragma omp parallel
    {
        int64_t* h = calloc((size_t)(n_bins + 2), sizeof(int64_t));
        double s1 = 0.0, s2 = 0.0;
#pragma omp for schedule(static)
        for (int64_t j = 0; j < n_blocks; ++j) {
            double z[4];
            oracle_normal_quad(seed, (uint32_t)(j % 1024), (uint32_t)(j / 1024), draw, layer, z);
            for (int k = 0; k < 4; ++k) {
                s1 += z[k];
                s2 += z[k] * z[k];
                int64_t b;
                if (z[k] < lo) b = 0;
                else if (z[k] >= hi) b = n_bins + 1;
                else {
                    b = 1 + (int64_t)floor((z[k] - lo) * scale);
                    if (b > n_bins) b = n_bins;
                }
                h[b] += 1;
            }
        }
#pragma omp critical
        {
            sums[0] += s1;
            sums[1] += s2;
            for (int32_t b = 0; b < n_bins + 2; ++b) hist[b] += h[b];
        }
        free(h);
    }
}

/* Batch of Philox blocks for arbitrary counters (n x 4 words in, n x 4 words and normals out). */
void oracle_philox_batch(const uint32_t* ctr, int64_t n, uint64_t seed, uint32_t* words,
                         double* normals)
{
    uint32_t key[2] = {(uint32_t)(seed & 0xffffffffu), (uint32_t)(seed >> 32)};
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) {
        uint32_t w[4];
        oracle_philox4x32_10(ctr + 4 * j, key, w);
        if (words) memcpy(words + 4 * j, w, sizeof w);
        if (normals) oracle_box_muller4(w, normals + 4 * j);
    }
}

/* Noise a_t^(i)[o] for a list of (t, i, o) triples (local indices; offsets added here). */
static double noise_at(uint64_t seed, uint32_t layer, uint32_t tg, uint32_t ig, int32_t o)
{
    double z[4];
    oracle_normal_quad(seed, (uint32_t)o >> 2, tg, ig, layer, z);
    return z[o & 3];
}

/*
 * Per-token quadratic readout loss of the noisy layer, absolute, for every draw:
 *   y_t = W x_t;  l_t^(i) = 1/2 || y_t + sigma a_t^(i) - u_t ||^2;  clean_t = 1/2 || y_t - u_t ||^2.
 * (noise equation of the page; the quadratic readout is the synthetic per-token loss.)
 * tokens: n_tok local token indices to evaluate (NULL: all N, n_tok = N).
 * loss: [K][n_tok], clean: [n_tok] (may be NULL).
 */
void oracle_noisy_linear_loss(const double* x, const double* W, const double* u, int64_t N,
                              int32_t d_in, int32_t d_out, int32_t K, double sigma,
                              uint64_t seed, uint32_t layer_id, uint32_t draw_offset,
                              uint32_t token_offset, const int64_t* tokens, int64_t n_tok,
                              double* loss, double* clean)
{
    if (!tokens) n_tok = N;
#pragma omp parallel
    {
        double* y = (double*)malloc(sizeof(double) * (size_t)d_out);
#pragma omp for schedule(dynamic, 4)
        for (int64_t j = 0; j < n_tok; ++j) {
            int64_t t = tokens ? tokens[j] : j;
            const double* xt = x + t * (int64_t)d_in;
            const double* ut = u + t * (int64_t)d_out;
            for (int32_t o = 0; o < d_out; ++o) {
                double acc = 0.0;
                const double* Wo = W + (int64_t)o * d_in;
                for (int32_t k = 0; k < d_in; ++k) acc += Wo[k] * xt[k];
                y[o] = acc;
            }
            if (clean) {
                double l = 0.0;
                for (int32_t o = 0; o < d_out; ++o) {
                    double e = y[o] - ut[o];
                    l += e * e;
                }
                clean[j] = 0.5 * l;
            }
            for (int32_t i = 0; i < K; ++i) {
                double l = 0.0;
                for (int32_t q = 0; 4 * q < d_out; ++q) {
                    double z[4];
                    oracle_normal_quad(seed, (uint32_t)q, token_offset + (uint32_t)t,
                                       draw_offset + (uint32_t)i, layer_id, z);
                    for (int32_t jj = 0; jj < 4 && 4 * q + jj < d_out; ++jj) {
                        int32_t o = 4 * q + jj;
                        double v = y[o] + sigma * z[jj] - ut[o];
                        l += v * v;
                    }
                }
                loss[(int64_t)i * n_tok + j] = 0.5 * l;
            }
        }
        free(y);
    }
}

/* Segment index of every token from cu_seqlens (cu[0] = 0, cu[n_seq] = N). */
static int32_t* segment_end_of(const int32_t* cu, int32_t n_seq, int64_t N)
{
    int32_t* end = (int32_t*)malloc(sizeof(int32_t) * (size_t)(N > 0 ? N : 1));
    for (int32_t s = 0; s < n_seq; ++s)
        for (int64_t t = cu[s]; t < cu[s + 1]; ++t) end[t] = cu[s + 1];
    return end;
}

/*
 * Centred loss and discounted credit, as written on the page:
 *   mean_t = (1/K) sum_i l_t^(i)     (the draw mean includes draw i itself)
 *   c_t^(i) = mean_t - l_t^(i)
 *   r_t^(i) = sum_{s = t}^{end(seg(t)) - 1} gamma^(s - t) c_s^(i)
 * computed as the explicit double sum (O(T^2) per segment).
 * loss, r: [K][N] row-major with leading dimension N.
 */
void oracle_credit(const double* loss, int32_t K, int64_t N, const int32_t* cu, int32_t n_seq,
                   double gamma, double* r)
{
    double* c = (double*)malloc(sizeof(double) * (size_t)(K * N > 0 ? K * N : 1));
    for (int64_t t = 0; t < N; ++t) {
        double m = 0.0;
        for (int32_t i = 0; i < K; ++i) m += loss[(int64_t)i * N + t];
        m /= (double)K;
        for (int32_t i = 0; i < K; ++i) c[(int64_t)i * N + t] = m - loss[(int64_t)i * N + t];
    }
    int32_t* end = segment_end_of(cu, n_seq, N);
#pragma omp parallel for schedule(dynamic, 16) collapse(2)
    for (int32_t i = 0; i < K; ++i) {
        for (int64_t t = 0; t < N; ++t) {
            double acc = 0.0, g = 1.0;
            for (int64_t s = t; s < end[t]; ++s) {
                acc += g * c[(int64_t)i * N + s];
                g *= gamma;
            }
            r[(int64_t)i * N + t] = acc;
        }
    }
    free(end);
    free(c);
}

/* Second route to the same credit: the backward recurrence r_t = c_t + gamma r_{t+1},
 * restarted at each segment end (used only to check the double sum). */
void oracle_credit_recurrence(const double* loss, int32_t K, int64_t N, const int32_t* cu,
                              int32_t n_seq, double gamma, double* r)
{
    for (int64_t t = 0; t < N; ++t) {
        double m = 0.0;
        for (int32_t i = 0; i < K; ++i) m += loss[(int64_t)i * N + t];
        m /= (double)K;
        for (int32_t i = 0; i < K; ++i) r[(int64_t)i * N + t] = m - loss[(int64_t)i * N + t];
    }
    for (int32_t i = 0; i < K; ++i)
        for (int32_t s = 0; s < n_seq; ++s)
            for (int64_t t = (int64_t)cu[s + 1] - 2; t >= cu[s]; --t)
                r[(int64_t)i * N + t] += gamma * r[(int64_t)i * N + t + 1];
}

/*
 * Output-error estimate (output-error equation of the page):
 *   g_t[o] = -(1 / (K_total sigma)) sum_{i < K_chunk} r_t^(i) a_t^(draw_offset + i)[o]
 * r: [K_chunk][N] (leading dimension N).  tokens / chans select the outputs (NULL: all).
 * g: [n_tok][n_ch].
 */
void oracle_output_error(const double* r, int32_t K_chunk, int32_t K_total, int64_t N,
                         int32_t d_out, double sigma, uint64_t seed, uint32_t layer_id,
                         uint32_t draw_offset, uint32_t token_offset, const int64_t* tokens,
                         int64_t n_tok, const int32_t* chans, int32_t n_ch, double* g)
{
    if (!tokens) n_tok = N;
    if (!chans) n_ch = d_out;
    const double scale = -1.0 / ((double)K_total * sigma);
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t j = 0; j < n_tok; ++j) {
        int64_t t = tokens ? tokens[j] : j;
        for (int32_t cc = 0; cc < n_ch; ++cc) {
            int32_t o = chans ? chans[cc] : cc;
            double acc = 0.0;
            for (int32_t i = 0; i < K_chunk; ++i)
                acc += r[(int64_t)i * N + t] *
                       noise_at(seed, layer_id, token_offset + (uint32_t)t,
                                draw_offset + (uint32_t)i, o);
            g[j * n_ch + cc] = scale * acc;
        }
    }
}

/*
 * Weight estimate (weight-estimate equation of the page), the explicit sum of outer
 * products over tokens:  G_W[o][k] = sum_t g_t[o] x_t[k].
 * g: [N][d_out], x: [N][d_in], GW: [d_out][d_in].
 */
void oracle_weight_grad(const double* g, const double* x, int64_t N, int32_t d_in,
                        int32_t d_out, double* GW)
{
#pragma omp parallel for schedule(static)
    for (int32_t o = 0; o < d_out; ++o) {
        double* row = GW + (int64_t)o * d_in;
        for (int32_t k = 0; k < d_in; ++k) row[k] = 0.0;
        for (int64_t t = 0; t < N; ++t) {
            double gt = g[t * d_out + o];
            const double* xt = x + t * (int64_t)d_in;
            for (int32_t k = 0; k < d_in; ++k) row[k] += gt * xt[k];
        }
    }
}

/*
 * Optimizer steps on the weight estimate (Dust page, section "설정": training with SGD and
 * momentum; section "Adam에서도 통할까?": the same estimate fed to Adam).  The page names the
 * optimizers only; these are their standard published forms:
 *   SGD with momentum (heavy ball, no dampening):  m <- mu m + G;  W <- W - lr m
 *   Adam (Kingma & Ba 2015, bias-corrected), step t >= 1:
 *     m <- b1 m + (1 - b1) G;  v <- b2 v + (1 - b2) G^2;
 *     W <- W - lr (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps)
 * Decoupled weight decay, when wd != 0, is applied first: W <- W - lr wd W.
 */
void oracle_sgd_momentum(double* W, double* m, const double* G, int64_t n, double lr, double mu,
                         double wd)
{
    for (int64_t j = 0; j < n; ++j) {
        W[j] -= lr * wd * W[j];
        m[j] = mu * m[j] + G[j];
        W[j] -= lr * m[j];
    }
}

void oracle_adam(double* W, double* m, double* v, const double* G, int64_t n, double lr,
                 double b1, double b2, double eps, double wd, int32_t t)
{
    const double c1 = 1.0 - pow(b1, (double)t);
    const double c2 = 1.0 - pow(b2, (double)t);
    for (int64_t j = 0; j < n; ++j) {
        W[j] -= lr * wd * W[j];
        m[j] = b1 * m[j] + (1.0 - b1) * G[j];
        v[j] = b2 * v[j] + (1.0 - b2) * G[j] * G[j];
        W[j] -= lr * (m[j] / c1) / (sqrt(v[j] / c2) + eps);
    }
}

/*
 * LM-head perturbation on cached logits (Dust page, section "간섭(interference) 줄이기",
 * third point: the LM head is perturbed directly on the cached logits; only the cross-entropy
 * is recomputed, on a slab of the vocabulary).  Reading: noise sigma a_t^(i)[v] is added to
 * the logits of the slab v in [v0, v0 + S) (channel index v, so the noise of a logit does not
 * depend on the slab); the per-token loss is the full-vocabulary cross-entropy
 *   l_t^(i) = log sum_v exp(z_t[v] + sigma a_t^(i)[v] [v in slab]) - (z_t[y_t] + sigma a_t^(i)[y_t] [y_t in slab]).
 * Computed as the plain definition in fp64 (max-shifted log-sum-exp).
 * z: [N][V], y: [N]; loss: [K][n_tok] absolute, clean: [n_tok] (unperturbed), tokens as above.
 */
void oracle_noisy_logits_ce(const double* z, const int32_t* y, int64_t N, int32_t V, int32_t v0,
                            int32_t S, int32_t K, double sigma, uint64_t seed, uint32_t layer_id,
                            uint32_t draw_offset, uint32_t token_offset, const int64_t* tokens,
                            int64_t n_tok, double* loss, double* clean)
{
    if (!tokens) n_tok = N;
#pragma omp parallel
    {
        double* zp = (double*)malloc(sizeof(double) * (size_t)V);
#pragma omp for schedule(dynamic, 4)
        for (int64_t j = 0; j < n_tok; ++j) {
            int64_t t = tokens ? tokens[j] : j;
            const double* zt = z + t * (int64_t)V;
            int32_t yt = y[t];
            double mx = zt[0];
            for (int32_t v = 1; v < V; ++v) mx = zt[v] > mx ? zt[v] : mx;
            double s = 0.0;
            for (int32_t v = 0; v < V; ++v) s += exp(zt[v] - mx);
            if (clean) clean[j] = mx + log(s) - zt[yt];
            for (int32_t i = 0; i < K; ++i) {
                for (int32_t v = 0; v < V; ++v) zp[v] = zt[v];
                for (int32_t v = v0; v < v0 + S; ++v)
                    zp[v] += sigma * noise_at(seed, layer_id, token_offset + (uint32_t)t,
                                              draw_offset + (uint32_t)i, v);
                double m2 = zp[0];
                for (int32_t v = 1; v < V; ++v) m2 = zp[v] > m2 ? zp[v] : m2;
                double s2 = 0.0;
                for (int32_t v = 0; v < V; ++v) s2 += exp(zp[v] - m2);
                loss[(int64_t)i * n_tok + j] = m2 + log(s2) - zp[yt];
            }
        }
        free(zp);
    }
}

/*
 * Attention-internal reward (Dust page, section "간섭(interference) 줄이기", second point):
 * a perturbation of the attention's internal projections (Q, K, V, gate) barely shows in
 * the token loss, so draw i is rewarded at token s by how well the output-error estimate at
 * the attention output, ghat_s, lines up with the change of that output under the draw:
 *   c_s^(i) = -<ghat_s, delta_o_s^(i)>.
 * The reward replaces the centred loss of the credit equation (no centring).
 * ghat: [N][d]; dO: [K][N][d] (draw-major); c: [K][N].
 */
void oracle_attn_reward(const double* ghat, const double* dO, int32_t K, int64_t N, int32_t d,
                        double* c)
{
#pragma omp parallel for schedule(static) collapse(2)
    for (int32_t i = 0; i < K; ++i) {
        for (int64_t t = 0; t < N; ++t) {
            double acc = 0.0;
            for (int32_t k = 0; k < d; ++k)
                acc += ghat[t * d + k] * dO[((int64_t)i * N + t) * d + k];
            c[(int64_t)i * N + t] = -acc;
        }
    }
}

/*
 * The credit equation applied to a given reward c (no centring):
 *   r_t^(i) = sum_{s = t}^{end(seg(t)) - 1} gamma^(s - t) c_s^(i)
 * as the explicit double sum.  c, r: [K][N].
 */
void oracle_discounted_credit(const double* c, int32_t K, int64_t N, const int32_t* cu,
                              int32_t n_seq, double gamma, double* r)
{
    int32_t* end = segment_end_of(cu, n_seq, N);
#pragma omp parallel for schedule(dynamic, 16) collapse(2)
    for (int32_t i = 0; i < K; ++i) {
        for (int64_t t = 0; t < N; ++t) {
            double acc = 0.0, g = 1.0;
            for (int64_t s = t; s < end[t]; ++s) {
                acc += g * c[(int64_t)i * N + s];
                g *= gamma;
            }
            r[(int64_t)i * N + t] = acc;
        }
    }
    free(end);
}

/*
 * SPSA / MeZO weight-space probe, the contrast estimator (thakicloud page, the SPSA paragraph:
 * two forwards, with the perturbation added and subtracted, estimate the gradient of every
 * parameter; gist.science 2605.15622 and the FedSPZO page: the perturbation is regenerated
 * from a shared seed, so only scalars travel).  Probe j moves the whole weight matrix along
 * z_j, drawn from the same generator in a separate counter space and stored at the weights'
 * precision (bf16):
 *   z_j[o][k] = bf16( normal of counter (k >> 2, o, probe_offset + j, layer_id | 2^31), index k & 3 )
 * The two perturbed forwards give
 *   L_+-^(j) = sum_t 1/2 || (W +- eps z_j) x_t - u_t ||^2,   p_j = (L_+ - L_-) / (2 eps),
 * and the weight estimate is (1/P_total) sum_j p_j z_j.
 */
static double bf16_round(double v)
{
    /* round to nearest, ties to even, at 8 significant bits (bf16 keeps fp32's exponent range) */
    if (v == 0.0) return 0.0;
    int e;
    frexp(v, &e);
    const double s = ldexp(1.0, 8 - e);
    return nearbyint(v * s) / s;
}

static double spsa_direction_at(uint64_t seed, uint32_t layer_id, uint32_t j, int32_t o, int32_t k)
{
    double z[4];
    oracle_normal_quad(seed, (uint32_t)k >> 2, (uint32_t)o, j, layer_id | 0x80000000u, z);
    return bf16_round(z[k & 3]);
}

/* z_j for j = probe_offset .. probe_offset + P - 1: Z [P][d_out][d_in]. */
void oracle_spsa_directions(uint64_t seed, uint32_t layer_id, uint32_t probe_offset, int32_t P,
                            int32_t d_out, int32_t d_in, double* Z)
{
#pragma omp parallel for collapse(2)
    for (int32_t j = 0; j < P; ++j)
        for (int32_t o = 0; o < d_out; ++o)
            for (int32_t k = 0; k < d_in; ++k)
                Z[((int64_t)j * d_out + o) * d_in + k] =
                    spsa_direction_at(seed, layer_id, probe_offset + (uint32_t)j, o, k);
}

/* p: [P]; Lp, Lm: [P] (may be NULL). */
void oracle_spsa_probe(const double* x, const double* W, const double* u, int64_t N, int32_t d_in,
                       int32_t d_out, int32_t P, double eps, uint64_t seed, uint32_t layer_id,
                       uint32_t probe_offset, double* p, double* Lp, double* Lm)
{
#pragma omp parallel
    {
        double* z = (double*)malloc(sizeof(double) * (size_t)d_out * (size_t)d_in);
#pragma omp for schedule(dynamic, 1)
        for (int32_t j = 0; j < P; ++j) {
            for (int32_t o = 0; o < d_out; ++o)
                for (int32_t k = 0; k < d_in; ++k)
                    z[(int64_t)o * d_in + k] =
                        spsa_direction_at(seed, layer_id, probe_offset + (uint32_t)j, o, k);
            double lp = 0.0, lm = 0.0;
            for (int64_t t = 0; t < N; ++t) {
                const double* xt = x + t * d_in;
                for (int32_t o = 0; o < d_out; ++o) {
                    double yp = 0.0, ym = 0.0;
                    for (int32_t k = 0; k < d_in; ++k) {
                        const double w = W[(int64_t)o * d_in + k], dz = eps * z[(int64_t)o * d_in + k];
                        yp += (w + dz) * xt[k];
                        ym += (w - dz) * xt[k];
                    }
                    const double ep = yp - u[t * d_out + o], em = ym - u[t * d_out + o];
                    lp += 0.5 * ep * ep;
                    lm += 0.5 * em * em;
                }
            }
            p[j] = (lp - lm) / (2.0 * eps);
            if (Lp) Lp[j] = lp;
            if (Lm) Lm[j] = lm;
        }
        free(z);
    }
}

/* G [d_out][d_in] = (1/P_total) sum_{j < P} p_j z_j. */
void oracle_spsa_estimate(const double* p, int32_t P, int32_t P_total, int32_t d_out, int32_t d_in,
                          uint64_t seed, uint32_t layer_id, uint32_t probe_offset, double* G)
{
#pragma omp parallel for schedule(static)
    for (int32_t o = 0; o < d_out; ++o)
        for (int32_t k = 0; k < d_in; ++k) {
            double acc = 0.0;
            for (int32_t j = 0; j < P; ++j)
                acc += p[j] * spsa_direction_at(seed, layer_id, probe_offset + (uint32_t)j, o, k);
            G[(int64_t)o * d_in + k] = acc / (double)P_total;
        }
}
