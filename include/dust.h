/*
 * dust.h: C ABI of libdust, a B200 (sm_100a) implementation of the Dust token-level
 * node-perturbation gradient estimator for one linear layer y_t = W x_t.
 *
 * The method (Dust review page, koala.ai.kr, "Dust: 역전파 없이 트랜스포머를 사전학습하다",
 * section "신용 할당(credit assignment): 보상에서 기울기까지"):
 *   noise equation          y_t -> y_t + sigma a_t,  a_t ~ N(0, I) independent per token, draw
 *   centred loss            c_s = mean_i(l_s^(i)) - l_s^(i)   (mean over the draws, self included)
 *   credit equation         r_t = sum_{s >= t} gamma^(s-t) c_s   (later tokens of the same sequence)
 *   output-error equation   g_t = -(1/(K sigma)) sum_i r_t^(i) a_t^(i)
 *   weight-estimate eq.     G_W = sum_t g_t x_t^T
 * The per-token loss computed by dust_noisy_linear_fwd is the quadratic readout
 * l_t = 1/2 || W x_t + sigma a_t - u_t ||^2.
 *
 * Noise is never stored: every kernel regenerates a_t^(i)[o] from a counter-based generator,
 * Philox4x32-10 (Salmon et al., SC'11) with Box-Muller.  The block with counter
 *     (o >> 2, token_offset + t, draw_offset + i, layer_id),  key (seed lo32, seed hi32)
 * gives four words w0..w3; with u(w) = (2 (w >> 9) + 1) 2^-24,
 *     z0 = rho cos(2 pi u(w1)), z1 = rho sin(2 pi u(w1)), rho = sqrt(-2 ln u(w0)),
 *     z2, z3 likewise from (w2, w3);  a_t^(i)[o] = z_{o & 3}.
 * Normals are fp32, within 1e-5 (absolute) of the exact value of the same formula.
 *
 * Conventions for every call:
 *   - Pointers named in the signature are DEVICE pointers unless said otherwise; arrays are
 *     row-major with a contiguous last dimension; pointers are 16-byte aligned.
 *   - The caller owns every buffer.  The library allocates no device memory; scratch space
 *     comes from the caller's workspace (size from dust_workspace_size).
 *   - Calls are asynchronous: they enqueue kernels on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream) and return after the launch.
 *   - Argument errors return synchronously and launch nothing.  Failures inside a kernel
 *     (a bounded wait that ran out) set a device error word that dust_last_device_error
 *     reads.  No C++ exception crosses this interface.
 *   - Sizes: N >= 1 tokens, 1 <= K.  bf16 layers need d_in and d_out multiples of 16;
 *     fp32 layers need d_out a multiple of 4.
 */
#ifndef DUST_H
#define DUST_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DUST_OK = 0,
    DUST_ERR_INVALID_ARG = 1,  /* a size, pointer, alignment or value is out of range       */
    DUST_ERR_UNSUPPORTED = 2,  /* valid, but outside what the kernels implement              */
    DUST_ERR_CUDA = 3,         /* a CUDA runtime call failed (launch, attribute, driver)     */
    DUST_ERR_TIMEOUT = 4,      /* a bounded device-side wait ran out (see dust_credit)       */
    DUST_ERR_WORKSPACE = 5     /* workspace pointer NULL, misaligned or smaller than needed  */
} dust_status;

typedef enum { DUST_F32 = 0, DUST_BF16 = 1 } dust_dtype;

typedef enum {
    DUST_OP_NOISY_LINEAR_FWD = 0,
    DUST_OP_CREDIT = 1,
    DUST_OP_WEIGHT_GRAD = 2,
    DUST_OP_LOGITS_CE = 3, /* d_in = vocabulary size V, d_out = slab size S */
    DUST_OP_SPSA_PROBE = 4 /* K = number of probes P */
} dust_op;

/* Identifies the noise of one call.  seed: generator key; layer_id: fourth counter word, so
 * layers draw independent noise; draw_offset: global index of the call's first draw (a
 * population larger than one call is processed in chunks); token_offset: global index of the
 * call's first token (a batch sharded over several GPUs keeps the same noise per token);
 * channel_offset: global index of the call's first output channel, a multiple of 4 (0 for a
 * whole layer; the slab start when only a slab of a layer's outputs is perturbed, as for the
 * LM head, so that a channel's noise does not depend on the slab). */
typedef struct {
    uint64_t seed;
    uint32_t layer_id;
    uint32_t draw_offset;
    uint32_t token_offset;
    uint32_t channel_offset;
} dust_noise_key;

/*
 * Noisy linear forward with the per-draw loss change (noise equation; quadratic readout).
 *   For each draw i in [0, K) and token t in [0, N):
 *     dloss[i * ld_dloss + t] = l_t^(i) - l_t^clean
 *                             = sum_o ( sigma a e_o + sigma^2 a^2 / 2 ),  a = a_t^(i)[o],
 *   with e = W x_t - u_t the clean residual.  The clean forward y = W x is computed once;
 *   the noise is added in the epilogue and never stored.
 * x: [N, d_in], W: [d_out, d_in], u: [N, d_out], all of dtype dt.
 * dloss: fp32 [K, ld_dloss], ld_dloss >= N.
 * workspace: dust_workspace_size(DUST_OP_NOISY_LINEAR_FWD, ...) bytes, 256-byte aligned.
 * Deterministic: the same inputs and key give bit-identical dloss.
 */
dust_status dust_noisy_linear_fwd(const void* x, const void* W, const void* u, dust_dtype dt,
                                  int64_t N, int32_t d_in, int32_t d_out, int32_t K,
                                  float sigma, dust_noise_key key, float* dloss,
                                  int64_t ld_dloss, void* workspace, size_t ws_bytes,
                                  void* stream);

/*
 * The perturbed layer outputs themselves, for callers that evaluate their own loss downstream
 * (for instance by recomputing the later blocks of a model for each draw, as the Dust page's
 * section "간섭(interference) 줄이기" describes for a perturbed block):
 *   y_out[(i * N + t) * ld_out + o] = (W x_t)[o] + sigma a_t^(i)[o],  i < K, t < N, o < d_out
 * with the same noise as dust_noisy_linear_fwd for the same key.  x [N, d_in], W [d_out, d_in]:
 * bf16 (d_in, d_out multiples of 16), 16-byte aligned.  y_out: DEVICE, out_dt fp32 or bf16
 * (rounded to nearest even), 16-byte aligned; ld_out >= d_out, a multiple of 16 bytes'
 * elements.  K N d_out values are written: this materialises what the fused forward never
 * stores.  Deterministic.
 */
dust_status dust_noisy_linear_output(const void* x, const void* W, dust_dtype dt, int64_t N,
                                     int32_t d_in, int32_t d_out, int32_t K, float sigma,
                                     dust_noise_key key, void* y_out, dust_dtype out_dt,
                                     int64_t ld_out, void* stream);

/*
 * LM-head perturbation on cached logits (Dust page, section "간섭(interference) 줄이기": the
 * LM head is perturbed on the cached logits and only the cross-entropy is recomputed, on a
 * slab of the vocabulary).  For each draw i and token t, with noise sigma a_t^(i)[v] added to
 * the logits of the slab v in [v0, v0 + S) (v is the noise channel; key.channel_offset must
 * be 0):
 *   dloss[i * ld_dloss + t] = CE(z_t + noise) - CE(z_t),  CE(z) = log sum_v exp(z_v) - z_{y_t},
 *                           = log(1 + X / E) - sigma a_t^(i)[y_t] [y_t in slab],
 *   E = sum_v exp(z_v - max z),  X = sum_{v in slab} exp(z_v - max z) (exp(sigma a) - 1).
 * z: logits [N, ld_z] of dtype dt (fp32 or bf16) with V valid columns; y: DEVICE int32 [N]
 * targets (a target outside [0, V) gives NaN for its token).  v0 and S multiples of 4,
 * v0 + S <= V.  The output feeds dust_credit, then dust_weight_grad with d_out = S and
 * key.channel_offset = v0 gives g on the slab and the slab's rows of the head weight estimate.
 * workspace: dust_workspace_size(DUST_OP_LOGITS_CE, dt, N, V, S, K) bytes.
 */
dust_status dust_noisy_logits_ce(const void* z, int64_t ld_z, dust_dtype dt, const int32_t* y,
                                 int64_t N, int32_t V, int32_t v0, int32_t S, int32_t K,
                                 float sigma, dust_noise_key key, float* dloss, int64_t ld_dloss,
                                 void* workspace, size_t ws_bytes, void* stream);

/*
 * Centred loss and discounted credit (centred-loss and credit equations).
 *   mean_t = (1/K) sum_i loss[i][t];  c = mean_t - loss[i][t];
 *   r[i][t] = c_t + gamma * r[i][t+1], restarted (r = c) at the last token of each segment.
 * loss: fp32 [K, ld_loss] (absolute losses or the dloss of dust_noisy_linear_fwd; the
 *       centring removes any per-token constant).  r: fp32 [K, ld_r].  ld_* >= N.
 * cu_seqlens: DEVICE int32 [n_seq + 1], non-decreasing, cu[0] = 0, cu[n_seq] = N; segment s
 *   is tokens [cu[s], cu[s+1]); credit never crosses a segment end.  Token N-1 always ends a
 *   segment.  Out-of-order entries give undefined r but no out-of-range access.
 * 0 <= gamma <= 1.  K >= 2 (with K = 1 the centred loss is identically 0).
 * The reverse scan chains token blocks by decoupled look-back.  Every wait is bounded (about
 * one second); a wait that runs out writes NaN to its block and sets DUST_ERR_TIMEOUT in the
 * device error word.  Bit-identical from call to call when no segment is longer than 8192
 * tokens (each block's carry is then composed from its successors' aggregates in a fixed
 * order); in a longer segment a block may take a successor's published inclusive value, and
 * the last bits can differ between calls.
 */
dust_status dust_credit(const float* loss, int64_t ld_loss, int32_t K, int64_t N,
                        const int32_t* cu_seqlens, int32_t n_seq, float gamma, float* r,
                        int64_t ld_r, void* workspace, size_t ws_bytes, void* stream);

/*
 * Attention-internal reward (Dust page, section "간섭(interference) 줄이기", second point): the
 * perturbations of an attention layer's internal projections (Q, K, V, gate) barely show in
 * the token loss, so each draw is rewarded by the alignment of the output-error estimate at
 * the attention output with the change that the draw caused there:
 *   c[i * ld_c + t] = -<ghat_t, delta_o_t^(i)>
 * ghat: fp32 [N, ld_g], the output-error estimate at the attention output (for instance the g
 *       of the output projection from dust_weight_grad); delta_o: [K, N, ld_delta_o] of dtype
 *       dt (draw-major; row (i, t) starts at (i * N + t) * ld_delta_o), the change of the
 *       attention output under draw i, computed by the caller's attention recomputation.
 * c: fp32 [K, ld_c], ld_c >= N.  16-byte aligned ghat and delta_o, ld_g a multiple of 4,
 * ld_delta_o and d multiples of 8 (bf16) or 4 (fp32); d <= 6144.  The reward feeds
 * dust_discounted_credit (no centring), then dust_weight_grad of the perturbed projection.
 * Deterministic (fixed-order sums).
 */
dust_status dust_attn_reward(const float* ghat, int64_t ld_g, const void* delta_o,
                             int64_t ld_delta_o, dust_dtype dt, int64_t N, int32_t d, int32_t K,
                             float* c, int64_t ld_c, void* stream);

/*
 * The credit equation on a given reward (no centring): r[i][t] = c[i][t] + gamma * r[i][t+1],
 * restarted at the last token of each segment.  Same arguments, layout, workspace
 * (dust_workspace_size(DUST_OP_CREDIT, ...)) and bounded waits as dust_credit; K >= 1.
 */
dust_status dust_discounted_credit(const float* c, int64_t ld_c, int32_t K, int64_t N,
                                   const int32_t* cu_seqlens, int32_t n_seq, float gamma,
                                   float* r, int64_t ld_r, void* workspace, size_t ws_bytes,
                                   void* stream);

/*
 * SPSA / MeZO weight-space probe, the contrast estimator (thakicloud page on zero-order
 * training, the SPSA paragraph: two forwards with a perturbation of all weights added and
 * subtracted; gist.science 2605.15622 and the FedSPZO page: the perturbation is regenerated
 * from a shared seed, so only scalars travel).  Probe j moves W along z_j [d_out, d_in]:
 *   z_j[o][k] = bf16 of the normal of counter (k >> 2, o, key.draw_offset + j,
 *               key.layer_id | 2^31), element k & 3 (the noise generator in its own space).
 * For each probe j in [0, P), with the quadratic readout l_t = 1/2 |y_t - u_t|^2:
 *   L_+-[j] = sum_t 1/2 |(W +- eps z_j) x_t - u_t|^2,   p[j] = (L_+[j] - L_-[j]) / (2 eps).
 * The two forwards share y = W x; they are evaluated through sum_t <W x_t - u_t, z_j x_t> and
 * sum_t |z_j x_t|^2, so p carries no cancellation error.
 * x [N, d_in], W [d_out, d_in], u [N, d_out]: bf16, 16-byte aligned; d_in and d_out multiples
 * of 16.  p: DEVICE fp32 [P]; L_plus, L_minus: optional DEVICE fp32 [P] (NULL to skip).
 * With tokens sharded over devices, p, L_plus and L_minus are sums over the local tokens:
 * summing them over the devices (P scalars each) gives the whole batch's values.
 * workspace: dust_workspace_size(DUST_OP_SPSA_PROBE, DUST_BF16, N, d_in, d_out, P) bytes.
 * key.token_offset and key.channel_offset must be 0 and key.layer_id below 2^31 (the top bit
 * marks the weight-space stream).  Deterministic.
 */
dust_status dust_spsa_probe(const void* x, const void* W, const void* u, dust_dtype dt, int64_t N,
                            int32_t d_in, int32_t d_out, int32_t P, float eps,
                            dust_noise_key key, float* p, float* L_plus, float* L_minus,
                            void* workspace, size_t ws_bytes, void* stream);

/*
 * The SPSA weight estimate: G (+)= (1 / P_total) sum_{j < P} p[j] z_j (z_j as in
 * dust_spsa_probe, regenerated from key).  p: DEVICE fp32 [P]; G: DEVICE fp32 [d_out, d_in],
 * 16-byte aligned; accumulate != 0 adds to G (probe chunks of one population).  d_in a
 * multiple of 4.  Deterministic (probes summed in order).
 */
dust_status dust_spsa_estimate(const float* p, int32_t P, int32_t P_total, int32_t d_in,
                               int32_t d_out, dust_noise_key key, float* G, int accumulate,
                               void* stream);

/*
 * Output-error estimate and weight estimate (output-error and weight-estimate equations).
 *   g_t[o] = -(1/(K_total sigma)) sum_{i < K_chunk} r[i][t] a_t^(draw_offset + i)[o]
 *   G_W[o][k] (+)= sum_t g_t[o] x_t[k]
 * r: fp32 [K_chunk, ld_r] holds the credit rows of draws key.draw_offset .. +K_chunk.
 * x: [N, d_in] of dtype dt.  G_W: fp32 [d_out, d_in]; accumulate != 0 adds to it (chunks of
 * one population), accumulate == 0 overwrites it.  g_out: optional fp32 [N, d_out] copy of g
 * (NULL to skip).  For bf16 x the contraction runs on the tensor cores with fp32
 * accumulation, and g enters it as g_terms bf16 terms:
 *   g_terms = 1: g rounded once to bf16 (relative rounding error up to 2^-9 per element;
 *                about 1.7e-3 relative Frobenius error of G_W when g is noise-dominated);
 *   g_terms = 2: hi = bf16(g) and lo = bf16(g - hi), both multiplied by x into the same
 *                accumulator (about 16 significant bits of g; twice the tensor-core work).
 * fp32 layers contract the fp32 g and accept either value.  2 N must fit in 31 bits.
 * Deterministic (split-K partials are reduced in a fixed order).  The workspace size does
 * not depend on g_terms.
 */
dust_status dust_weight_grad(const float* r, int64_t ld_r, const void* x, dust_dtype dt,
                             int64_t N, int32_t d_in, int32_t d_out, int32_t K_chunk,
                             int32_t K_total, float sigma, dust_noise_key key, float* G_W,
                             int accumulate, float* g_out, int32_t g_terms, void* workspace,
                             size_t ws_bytes, void* stream);

/*
 * dust_credit without a caller workspace (the paper has no counterpart: this is a packaging
 * variant for callers that cannot allocate device memory, for example a plugin run by a host
 * engine that owns every buffer and forbids allocation while it executes, or a process under a
 * fixed memory budget).  Same arguments, result and errors as dust_credit, minus the
 * workspace: the look-back scratch lives in a 4 MiB static device array of the library, which
 * every device that loads the library holds until the process exits.  The call allocates
 * nothing (no cudaMalloc, no allocating library routine).
 *   - Sizes whose scratch exceeds 4 MiB are rejected with DUST_ERR_WORKSPACE.  The scratch is
 *     exactly dust_workspace_size(DUST_OP_CREDIT, DUST_F32, N, 0, 0, K) bytes, so a caller
 *     checks a size by comparing that value with 4 MiB (4194304).  For K <= 128 it is
 *     about 16 K bytes per 128 tokens plus 256, so K = 32 allows N up to about 1.05 million
 *     tokens and K = 64 about 520,000.  For K > 128 the draws form ceil(K / 128) groups of
 *     up to 128 rows, each with its own look-back state, plus a 4 N byte per-token mean:
 *     K = 256 allows N up to about 116,000 tokens.
 *   - The first call on a device (and the first after that device's context was reset) looks
 *     up the array's device address, with that device current; make that first call before
 *     any stream capture.  Concurrent first calls from several host threads are safe.
 *   - Every call shares the one array, and the ticket and flags are cleared on `stream` before
 *     each launch.  Calls whose kernels overlap on the GPU (other streams, other threads)
 *     race on the scratch and give wrong results: serialize them.
 */
dust_status dust_credit_no_alloc(const float* loss, int64_t ld_loss, int32_t K, int64_t N,
                                 const int32_t* cu_seqlens, int32_t n_seq, float gamma,
                                 float* r, int64_t ld_r, void* stream);

/*
 * Optimizer step on a weight estimate.  The Dust page trains with SGD and momentum (section
 * "설정") and reports the same estimate fed to Adam (section "Adam에서도 통할까?"); it names
 * the optimizers only, so their standard published forms are used, with decoupled weight
 * decay applied first (W <- W - lr wd W):
 *   DUST_OPT_SGD_MOMENTUM:  m <- momentum m + G;  W <- W - lr m
 *   DUST_OPT_ADAM (Kingma & Ba, bias-corrected, step t >= 1):
 *     m <- b1 m + (1 - b1) G;  v <- b2 v + (1 - b2) G^2;
 *     W <- W - lr (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps)
 * All state is fp32 and updated in place.
 */
typedef enum { DUST_OPT_SGD_MOMENTUM = 1, DUST_OPT_ADAM = 2 } dust_opt_kind;

typedef struct {
    int32_t kind;        /* dust_opt_kind */
    int32_t step;        /* Adam: 1-based step count t */
    float lr;            /* >= 0 */
    float momentum;      /* SGD: 0 <= momentum < 1 */
    float beta1, beta2;  /* Adam: 0 <= beta < 1 */
    float eps;           /* Adam: > 0 */
    float weight_decay;  /* >= 0, decoupled */
} dust_opt_params;

/* One step on n elements: G (read), W fp32 master weights, m (and v for Adam) state, all
 * DEVICE fp32 [n], 16-byte aligned, updated in place; W_bf16 (DEVICE, optional, NULL to skip)
 * receives the updated W rounded to bf16 (for the next forward).  `opt` is a HOST pointer. */
dust_status dust_optimizer_step(const dust_opt_params* opt, const float* G, float* W,
                                void* W_bf16, float* m, float* v, int64_t n, void* stream);

/* dust_weight_grad with the optimizer step fused into the pass that finishes G_W (the
 * contraction's epilogue, or the split-K reduction): the weight estimate is not written and
 * read back before the step.  Same arguments as dust_weight_grad (bf16 only), plus the step:
 * W, W_bf16, m, v as in dust_optimizer_step with n = d_out * d_in.  G_W may be NULL (then it
 * is not stored; accumulate must be 0).  The result equals dust_weight_grad followed by
 * dust_optimizer_step. */
dust_status dust_weight_grad_step(const float* r, int64_t ld_r, const void* x, dust_dtype dt,
                                  int64_t N, int32_t d_in, int32_t d_out, int32_t K_chunk,
                                  int32_t K_total, float sigma, dust_noise_key key, float* G_W,
                                  int accumulate, float* g_out, int32_t g_terms,
                                  const dust_opt_params* opt, float* W, void* W_bf16, float* m,
                                  float* v, void* workspace, size_t ws_bytes, void* stream);

/*
 * Grouped forms: the same three steps for many bf16 layers that share the token batch
 * (N tokens, the same sequences, K, sigma, seed), one kernel launch per step for up to 64
 * layers (more layers take more launches).  A transformer block stack perturbs each linear
 * layer on its own (Dust page, section "간섭 줄이기": each block and layer type is perturbed
 * separately with its own noise), so each layer has its own noise (its layer_id) and its own
 * per-token loss.  Grouping fills the GPU when single layers are too small to.
 * `layers` is a HOST array of n_layers descriptors; the pointers inside are DEVICE pointers.
 * Per layer: x [N, d_in], W [d_out, d_in], u [N, d_out] (bf16; d_in, d_out multiples of 16);
 * dloss fp32 [K, ld_dloss]; r fp32 [K, ld_r]; G_W fp32 [d_out, d_in]; g_out optional fp32
 * [N, d_out].  key.layer_id is ignored (each descriptor's layer_id is used).  The workspace is
 * dust_workspace_size_grouped bytes; each layer gets its own region.  dloss and r equal the
 * single-layer calls bit for bit; G_W can differ by rounding, because the split of the token
 * sum (split-K) is chosen for the whole group.
 */
typedef struct {
    const void* x;
    const void* W;
    const void* u;
    int32_t d_in, d_out;
    uint32_t layer_id;
    uint32_t reserved; /* must be 0 */
    float* dloss;
    int64_t ld_dloss;
    float* r;
    int64_t ld_r;
    float* G_W;
    float* g_out;
} dust_layer_desc;

/* dust_noisy_linear_fwd for every layer: reads x, W, u; writes dloss. */
dust_status dust_noisy_linear_fwd_grouped(const dust_layer_desc* layers, int32_t n_layers,
                                          int64_t N, int32_t K, float sigma, dust_noise_key key,
                                          void* workspace, size_t ws_bytes, void* stream);
/* dust_credit for every layer: reads dloss, writes r (cu_seqlens shared by all layers). */
dust_status dust_credit_grouped(const dust_layer_desc* layers, int32_t n_layers, int32_t K,
                                int64_t N, const int32_t* cu_seqlens, int32_t n_seq, float gamma,
                                void* workspace, size_t ws_bytes, void* stream);
/* dust_weight_grad for every layer: reads r (K_chunk rows) and x; writes (or adds to) G_W and,
 * where not NULL, g_out; g_terms (1 or 2) as in dust_weight_grad, for every layer. */
dust_status dust_weight_grad_grouped(const dust_layer_desc* layers, int32_t n_layers, int64_t N,
                                     int32_t K_chunk, int32_t K_total, float sigma,
                                     dust_noise_key key, int accumulate, int32_t g_terms,
                                     void* workspace, size_t ws_bytes, void* stream);
/* Workspace bytes of a grouped call of step `op`. */
size_t dust_workspace_size_grouped(dust_op op, const dust_layer_desc* layers, int32_t n_layers,
                                   int64_t N, int32_t K);

/* Workspace bytes that `op` needs for these sizes (0 if none).  d_in / d_out are ignored by
 * DUST_OP_CREDIT, K by DUST_OP_WEIGHT_GRAD. */
size_t dust_workspace_size(dust_op op, dust_dtype dt, int64_t N, int32_t d_in, int32_t d_out,
                           int32_t K);

/* Static, NUL-terminated name of a status code. */
const char* dust_status_string(dust_status s);

/* Synchronizes `stream`, then reads and clears the device error word of the current device:
 * DUST_OK if no kernel reported a failure since the last read.  *info (if not NULL) receives
 * the failing block index or wait site recorded with the error. */
dust_status dust_last_device_error(void* stream, int32_t* info);

/* Profiling.  While enabled, every kernel that libdust launches is bracketed by two CUDA
 * events on its stream (cheap; no synchronization).  dust_profile_read synchronizes the
 * device, then returns up to `max` records (static kernel name, duration in ms) in launch
 * order and clears them.  At most `capacity` launches are kept; later ones are dropped.
 * Host-side state is one global list (not thread-safe). */
dust_status dust_profile_enable(int32_t capacity);
void dust_profile_disable(void);
int32_t dust_profile_read(const char** names, float* ms, int32_t max);

/* Test support: the generator on its own.  ctr: DEVICE uint32 [n, 4] counters; the key is
 * (seed lo32, seed hi32).  Writes DEVICE words [n, 4] and fp32 normals [n, 4] (either may be
 * NULL).  Uses the same device functions as the estimator kernels. */
dust_status dust_debug_philox(const uint32_t* ctr, int64_t n, uint64_t seed, uint32_t* words,
                              float* normals, void* stream);

/* Test and measurement support: the generator's throughput ceiling.  out[g] (DEVICE fp32
 * [n]) = the sum of the normals a_t^(i)[o] of token t = key.token_offset + g, draw
 * i = key.draw_offset, layer key.layer_id, channels o = key.channel_offset + 0 .. 4 n_quads - 1
 * (the estimator's mapping).  The kernel only generates and adds (one add per normal), so
 * its rate bounds what the noise kernels can reach.  key.channel_offset a multiple of 4. */
dust_status dust_debug_normal_sum(dust_noise_key key, int64_t n, int32_t n_quads, float* out,
                                  void* stream);

/* Measurement support: the generator's integer part alone.  out[g] (DEVICE uint32 [n]) = the
 * XOR of the four Philox4x32-10 words of every block (key.channel_offset / 4 + j,
 * key.token_offset + g, key.draw_offset, key.layer_id), j < n_blocks, under the estimator's
 * key.  Its rate (4 n n_blocks words per launch) shows what the widening multiplies alone
 * allow the noise kernels.  key.channel_offset a multiple of 4; out 4-byte aligned. */
dust_status dust_debug_word_sum(dust_noise_key key, int64_t n, int32_t n_blocks, uint32_t* out,
                                void* stream);

/* Test support: the next dust_credit launch on any stream skips publishing the look-back
 * status of token block `block` (-1: none), so that the block before it waits until its
 * bounded wait runs out.  Used to test the timeout path; never set in normal use. */
void dust_debug_credit_skip_publish(int32_t block);

/* Test support: the form the bf16 forward (dust_noisy_linear_fwd and its grouped form) takes
 * for N tokens, K draws and n_layers layers of output widths d_out[0 .. n_layers-1] (HOST
 * int32) on a device with `sms` SMs.  *persistent = 1: one CTA per SM walks a balanced range
 * of (tile, draw, channel half) items (*split = 0); 0: one 128 x 256 tile per CTA, two CTAs per
 * SM, each tile of the last, partial wave cut into *split unit ranges.  Host-only: touches no
 * device.  DUST_ERR_INVALID_ARG on a non-positive size or a NULL pointer. */
dust_status dust_debug_fwd_plan(int64_t N, int32_t K, int32_t n_layers, const int32_t* d_out,
                                int32_t sms, int32_t* persistent, int32_t* split);

#ifdef __cplusplus
}
#endif

#endif /* DUST_H */
