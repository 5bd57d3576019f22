/*
 * dgen -- per-step canvas denoising of a uniform-state discrete-diffusion MoE
 * language model on one NVIDIA B200 (sm_100a).  C ABI.
 *
 * The method (DiffusionGemma; hyper.ai digest of the paper, Method): a prompt
 * goes through the causal encoder to build a KV cache (three-stage pipeline,
 * stage 1); a noisy 256-token canvas is then refined for T steps by the
 * decoder, which attends bidirectionally over the canvas and to the cache
 * (stage 2; eq. 3 gives the logits L_t), followed by the sampler (eq. 4:
 * tempered softmax, then the Step that commits confident tokens and renoises
 * the rest uniformly; alphasignal.ai article, "How text diffusion actually
 * works", step 2).
 *
 * Conventions, for every entry point:
 *  - All device pointers are plain CUDA device addresses on the handle's
 *    device.  Weights are bf16 (IEEE bfloat16 bit patterns), row-major, and
 *    are OWNED BY THE CALLER: they must stay valid and unchanged for the life
 *    of the handle.  The library owns the KV cache, the canvas state and all
 *    scratch, and frees them in dgen_destroy.
 *  - Calls are asynchronous on the handle's stream (given at create) unless
 *    stated; they enqueue work and return.  Output buffers are valid once the
 *    stream reaches the call (e.g. after dgen_synchronize).
 *  - Every call returns DGEN_OK (0) or a negative status; nothing is enqueued
 *    when a call fails its argument checks.  A device-side check (a bounded
 *    wait that ran out) records DGEN_EDEVICE, reported by dgen_synchronize.
 *  - There is no CPU fallback: every step of the path runs in this library's
 *    CUDA kernels.
 */
#ifndef DGEN_H
#define DGEN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DGEN_OK 0
#define DGEN_EINVAL (-1)  /* bad argument or unsupported shape */
#define DGEN_ENOMEM (-2)  /* device allocation failed */
#define DGEN_ECAP (-3)    /* prompt longer than prompt_max */
#define DGEN_ECUDA (-4)   /* a CUDA runtime/driver call failed */
#define DGEN_EDEVICE (-5) /* a device-side bounded wait ran out (see dgen_synchronize) */
#define DGEN_ESTATE (-6)  /* call out of order (e.g. a step before the prompt cache exists) */
#define DGEN_ESCRATCH (-7) /* sizes exceed the fixed scratch of dgen_sample_from_logits_noalloc */

/* Model shape and run settings.  The workload descriptions fix the shapes;
 * the pages fix C = 256 (Key Contributions) and tau 0.8 -> 0.4 (Method,
 * sampler paragraph).  Requirements checked at create: d_model, expert_width,
 * shared_width and n_q_heads*head_dim multiples of 64; d_model a multiple of
 * 128 and at most 4096; head_dim in {64, 128, 256}; n_q_heads a multiple of n_kv_heads;
 * top_k <= n_experts <= 256, top_k <= 16; canvas <= 1024; vocab a multiple of
 * 256 and < 2^31; shared_width <= 8 expert_width; batch * max(canvas,
 * prompt_max) token rows within what one routing launch takes (SM count x
 * min(1024, 8192 / top_k)).
 *
 * expert_fp8 = 1 (the pages' speeds are for FP8: hyper.ai digest, Experiment;
 * alphasignal.ai, "Architecture"): at create the library quantizes every expert
 * and shared-FFN weight matrix to OCP FP8 E4M3 (round to nearest even) with one
 * power-of-two scale per stored row, into memory it owns (about half the bf16
 * size; the caller's bf16 weights must still stay valid); in each MoE block the
 * normed token rows and the gated activations are quantized the same way per
 * token row, the expert GEMMs run on the tensor cores' E4M3 path with fp32
 * accumulation, and the epilogues multiply by the two row scales.  Router,
 * gates, attention and the LM head stay bf16.
 *
 * self_cond_width = w_sc > 0 (a multiple of 64) turns on self-conditioning
 * (hyper.ai digest, Method, eqs. 3-4): every decoder pass also computes the
 * next step's state z = FFW(p0_hat E), p0_hat = Softmax(L_t / tau_s) rounded
 * to bf16, E the embedding, FFW a pre-RMSNorm gated-GELU FFN d -> w_sc -> d
 * (weights in dgen_weights), and the next pass adds z to the canvas token
 * embeddings.  z is zero at the first step of a block: dgen_init_canvas,
 * dgen_set_canvas, dgen_prefill_prompt, dgen_set_prompt_kv and
 * dgen_append_canvas clear it (dgen_set_self_cond sets it).  0 = off (z = 0). */
typedef struct dgen_config {
    int32_t n_layers;
    int32_t d_model;
    int32_t n_q_heads;
    int32_t n_kv_heads;
    int32_t head_dim;
    int32_t n_experts;
    int32_t top_k;
    int32_t expert_width;  /* w: width of each routed gated-GELU expert */
    int32_t shared_width;  /* ws: width of the shared dense gated FFN, 0 = none */
    int32_t vocab;         /* V; the LM head is tied to the embedding */
    int32_t batch;         /* B independent sequences, one canvas each */
    int32_t prompt_max;    /* capacity of the prompt part of the KV cache */
    int32_t canvas;        /* C canvas tokens per sequence */
    int32_t commit_per_step; /* tokens committed per step; 0 -> ceil(C / T) */
    float tau_max;         /* 0.8 */
    float tau_min;         /* 0.4 */
    float rms_eps;         /* 1e-6 */
    float rope_base;       /* 10000 */
    int32_t expert_fp8;    /* 1: the routed experts and the shared FFN run in FP8 E4M3 (see below), 0: bf16 */
    int32_t self_cond_width; /* w_sc of the self-conditioning FFW (see above), 0 = no self-conditioning */
} dgen_config;

/* Per-layer weights (bf16, row-major, caller-owned device memory).
 * Each GEMM weight is stored [out][in] ("K-major"). */
typedef struct dgen_layer_weights {
    const void* attn_norm;        /* [d]                      gain g, applied as (1 + g) */
    const void* w_qkv;            /* [(Hq + 2 Hkv) hd][d]     rows: q heads, k heads, v heads */
    const void* w_o;              /* [d][Hq hd] */
    const void* ffn_norm;         /* [d] */
    const void* w_router;         /* [E][d] */
    const void* w_gate_up;        /* [E][2w][d]               gate and up rows interleaved in blocks
                                   *  of 16: rows 32j..32j+15 = gate features 16j..16j+15,
                                   *  rows 32j+16..32j+31 = up features 16j..16j+15 */
    const void* w_down;           /* [E][d][w] */
    const void* w_shared_gate_up; /* [2 ws][d]  same interleaving; NULL when shared_width == 0 */
    const void* w_shared_down;    /* [d][ws]    or NULL when shared_width == 0 */
} dgen_layer_weights;

typedef struct dgen_weights {
    const void* embed;                /* [V][d] token embedding E, also the LM head */
    const void* final_norm;           /* [d] */
    const dgen_layer_weights* layers; /* host array of n_layers entries, copied at create */
    /* the self-conditioning FFW (read only when self_cond_width > 0, else may be NULL) */
    const void* sc_norm;              /* [d]          pre-norm gain, applied as (1 + g) */
    const void* w_sc_gate_up;         /* [2 w_sc][d]  gate and up rows interleaved in blocks of 16 */
    const void* w_sc_down;            /* [d][w_sc] */
} dgen_weights;

typedef struct dgen_handle dgen_handle;

/* Validates the config, records the weight pointers (no copy), allocates the
 * KV cache, canvas state and scratch on the current device, builds the TMA
 * descriptors.  stream: a cudaStream_t (NULL = legacy default stream).
 * Synchronous.  Errors: EINVAL (shape), ENOMEM, ECUDA. */
int dgen_create(const dgen_config* cfg, const dgen_weights* weights, void* stream, dgen_handle** out);

/* Waits for the stream, frees everything the handle owns.  NULL is a no-op. */
int dgen_destroy(dgen_handle* h);

/* Stage 1 of the pipeline (hyper.ai digest, Method, three-stage pipeline):
 * the causal encoder pass over prompt_dev [B][P] (int32 token ids in [0, V))
 * writes K (after RoPE, positions 0..P-1) and V of every layer into the cache.
 * Errors: EINVAL (P < 1), ECAP (P > prompt_max). */
int dgen_prefill_prompt(dgen_handle* h, const int32_t* prompt_dev, int32_t P);

/* Loads a precomputed bf16 prompt cache for one layer instead of running the
 * prompt pass (the long-prompt workload's "prompt KV cache precomputed in
 * bf16").  k_dev, v_dev: [B][Hkv][P][hd], K already rotated for positions
 * 0..P-1.  Copied into the library's cache.  The cache counts as built once
 * every layer has been loaded with the same P.  Errors: EINVAL, ECAP. */
int dgen_set_prompt_kv(dgen_handle* h, int32_t layer, const void* k_dev, const void* v_dev, int32_t P);

/* Draws the initial noisy canvas x[b][i] = uniform token from
 * Philox4x32-10(key = seed; counter = (o + i, 0, b, 0)), lane 0, mapped to [0, V)
 * by floor(word * V / 2^32) (alphasignal.ai article, step 1 "canvas
 * initialization"); clears every committed flag.  o = 0 for the first block
 * after the prompt, (canvases appended since) x C after dgen_append_canvas. */
int dgen_init_canvas(dgen_handle* h, uint64_t seed);

/* Teacher forcing: overwrite the canvas state with tok_dev [B][C] int32 and
 * committed_dev [B][C] uint8 (0/1).  committed_dev may be NULL (all 0). */
int dgen_set_canvas(dgen_handle* h, const int32_t* tok_dev, const uint8_t* committed_dev);

/* Copies the canvas state out (either pointer may be NULL). */
int dgen_get_canvas(const dgen_handle* h, int32_t* tok_dev, uint8_t* committed_dev);

/* One decoder pass L_t = Decoder(x_t, z_t, H) (hyper.ai digest, Method,
 * eq. 3) over all B canvases, at step s of T (z_t = 0 without
 * self-conditioning, else the state the previous pass left): non-causal attention of the
 * canvas (positions P..P+C-1) over [prompt cache ; canvas], the top-k routed
 * MoE (+ shared FFN), the final norm and the tied LM head, whose epilogue
 * reduces each row to the statistics of Softmax(L_t / tau_s) (eq. 4, first
 * line) with tau_s = tau_min + (tau_max - tau_min)(1 - s/T).
 * logits_dev_or_null: if not NULL (16-byte aligned, else EINVAL), also stores
 * the fp32 logits [B][C][V].
 * With self-conditioning the pass then computes z_{t - dt} = FFW(p0_hat E)
 * (eq. 4, second line) for every canvas position, committed or not, as the
 * next pass's state.
 * Errors: EINVAL (s, T), ESTATE (no prompt cache). */
int dgen_denoise_step(dgen_handle* h, int32_t s, int32_t T, float* logits_dev_or_null);

/* Sets the self-conditioning state the next dgen_denoise_step adds to the
 * canvas embeddings: z_dev [B][C][d] fp32 (copied), or NULL for z = 0.
 * Errors: EINVAL (self_cond_width == 0 and z_dev not NULL). */
int dgen_set_self_cond(dgen_handle* h, const float* z_dev_or_null);

/* The sampler after dgen_denoise_step (or dgen_set_logits) of the same s, T:
 * per position, conf = log max_v Softmax(L / tau_s) and the argmax (ties ->
 * lowest v); per canvas, the m = min(commit, #uncommitted) uncommitted
 * positions of highest conf (ties -> lower position) are set to their argmax
 * and frozen (m = #uncommitted at s = T-1); every other uncommitted position is
 * redrawn uniformly from Philox4x32-10(seed; (o + i, s, b, 1)), lane 0 (o as in
 * dgen_init_canvas).
 * conf_dev_or_null: if not NULL, receives conf [B][C] fp32. */
int dgen_sample_commit(dgen_handle* h, int32_t s, int32_t T, uint64_t seed, float* conf_dev_or_null);

/* The pages' own sampler (hyper.ai digest of the DiffusionGemma paper, Method:
 * entropy-bounded sampler with adaptive stopping).  Tempering uses tau of step s
 * of a budget of T_max steps.  Per position: the entropy H of Softmax(L / tau)
 * (natural log; written to entropy_dev_or_null [B*C] when given) and the argmax.
 *   logits_dev_or_null == NULL: from the LM head's statistics of the last
 *     dgen_denoise_step, which must have been called with the same s and T_max
 *     (the production path: no stored logits);
 *   else: from the given fp32 logits [B*C][V] (16-byte aligned, else EINVAL),
 *     tempered through a 1/tau word of its own, so the statistics that
 *     dgen_sample_commit reads are neither used nor changed.
 * Per canvas the candidate positions -- the uncommitted ones when freeze = 1,
 * every position when freeze = 0 (earlier choices may be revised) -- rank by
 * (H, position); the longest prefix whose mutual-information bound (sum of the
 * prefix's entropies minus the largest; the first position always passes) stays
 * below gamma takes its argmax (committed flag 1); every other candidate is
 * redrawn from the same Philox stream as dgen_sample_commit (committed flag 0).
 * Stop test for s > 0: mean H over the canvas below stop_threshold and the
 * argmax canvas equal to the one of this handle's previous step; on a stop or at
 * s = T_max - 1 every candidate takes its argmax.  A canvas that stopped (or,
 * with freeze = 1, has every position committed) is done and later steps of the
 * block (s > 0) leave it unchanged.  stop_dev_or_null [B] uint8 receives the
 * stop flags.  gamma, stop_threshold >= 0; freeze 0 or 1. */
int dgen_sample_commit_eb(dgen_handle* h, const float* logits_dev_or_null, int32_t s, int32_t T_max, uint64_t seed,
                          float gamma, float stop_threshold, int32_t freeze, float* entropy_dev_or_null,
                          uint8_t* stop_dev_or_null);

/* One block with the entropy-bounded sampler and adaptive stopping (same page,
 * Method: sampler paragraph and adaptive stopping; Experiment: at most 48 steps):
 * prompt pass over prompt_dev [B][P] (prompt_dev NULL: none, the block continues
 * from the cache as it is, e.g. after dgen_append_canvas; P is then ignored;
 * ESTATE without a cache), initial canvas, then for s = 0, 1, ...:
 * dgen_denoise_step(s, T_max) + dgen_sample_commit_eb(NULL logits); after each
 * step the host reads the per-canvas done flags (one small device-to-host copy
 * and a stream synchronisation) and stops launching once every canvas is done,
 * at the latest after T_max steps.  Copies the canvas to out_dev [B][C] and the
 * number of steps each canvas took to steps_host [B] (host memory).
 * Synchronous. */
int dgen_generate_block_eb(dgen_handle* h, const int32_t* prompt_dev, int32_t P, int32_t T_max, uint64_t seed,
                           float gamma, float stop_threshold, int32_t freeze, int32_t* out_dev, int32_t* steps_host);

/* Stage 3 of the pipeline (hyper.ai digest, Method, three-stage pipeline):
 * the current canvas [B][C] goes through the causal encoder at positions
 * P..P+C-1 (query i sees the cache and canvas keys up to P + i) and its K / V
 * are appended to the cache, which then holds P + C positions; the next block's
 * Philox draws start at canvas position (blocks appended) x C.  The prompt
 * pass's routing teacher forcing (dgen_force_routing) applies to this pass too.
 * Errors: ESTATE (no cache), ECAP (P + C > prompt_max). */
int dgen_append_canvas(dgen_handle* h);

/* Block-autoregressive generation (same page, Method: the model denoises one
 * 256-token canvas at a time and commits it to the sequence history before the
 * next): prompt pass over prompt_dev [B][P], then n_blocks times (initial canvas,
 * T x (dgen_denoise_step + dgen_sample_commit), dgen_append_canvas except after
 * the last block).  out_dev [B][n_blocks * C] receives each sequence's blocks
 * in order.  Errors: ECAP (P + (n_blocks - 1) C > prompt_max). */
int dgen_generate(dgen_handle* h, const int32_t* prompt_dev, int32_t P, int32_t n_blocks, int32_t T, uint64_t seed,
                  int32_t* out_dev);

/* Replaces the LM head's output for the next dgen_sample_commit by the fp32
 * logits [B][C][V] at logits_dev (reduced with tau_s of step s of T).  For
 * testing the sampler on given logits. */
int dgen_set_logits(dgen_handle* h, const float* logits_dev, int32_t s, int32_t T);

/* One whole block: prompt pass over prompt_dev [B][P], initial canvas, then
 * T x (dgen_denoise_step + dgen_sample_commit); copies the final canvas to
 * out_dev [B][C] int32. */
int dgen_generate_block(dgen_handle* h, const int32_t* prompt_dev, int32_t P, int32_t T, uint64_t seed,
                        int32_t* out_dev);

/* Same as dgen_generate_block with HOST buffers: prompt_host [B][P] is copied
 * to the device, the block is generated, and the canvas is copied back into
 * out_host [B][C].  Synchronous (returns after out_host is written). */
int dgen_generate_block_host(dgen_handle* h, const int32_t* prompt_host, int32_t P, int32_t T, uint64_t seed,
                             int32_t* out_host);

/* The uniform-state forward process (hyper.ai digest, Method, eq. 1) on
 * x0_dev [B][C]: x_t[b][i] = x0 if lane 1 of Philox4x32-10(seed; (i, step, b, 2))
 * is below floor(kappa * 2^32), else the uniform token of lane 0.  Writes
 * xt_dev [B][C].  For building teacher-forced canvases. */
int dgen_forward_noise(dgen_handle* h, const int32_t* x0_dev, float kappa, uint64_t seed, int32_t step,
                       int32_t* xt_dev);

/* Waits for the handle's stream; returns DGEN_EDEVICE if a device-side bounded
 * wait ran out since the last call (and clears the flag), DGEN_ECUDA on a CUDA
 * error, else DGEN_OK. */
int dgen_synchronize(dgen_handle* h);

/* Number of kernels this handle has launched so far (for launch accounting). */
int64_t dgen_launch_count(const dgen_handle* h);

/* Tuning overrides (value 0 = the automatic choice).  DGEN_TUNE_EXPERT_CHUNK:
 * token-chunk width of the grouped expert GEMMs (32, 64, 128 or 256).
 * DGEN_TUNE_ATTN_SPLITS: key splits of the decoder's attention (<= 32).
 * DGEN_TUNE_ROUTER_SPLITS: K splits per row tile of the router GEMM.
 * DGEN_TUNE_QKV_SPLITS: K splits of the QKV projection (1 = none, <= 4).
 * DGEN_TUNE_ATTN_KERNEL: 1 = run attention (canvas pass and the causal prompt
 * and append passes) on the warp-level mma.sync kernel instead of the tcgen05
 * kernel.  For measurement; results do not depend on them except for the order
 * of fp32 sums.  DGEN_TUNE_ROUTE_BARRIER_EXTRA (test hook, 0 or 1): 1 raises
 * the target of the routing launch's grid barrier by one, so that its bounded
 * wait runs out (about 2 s): the pass records DGEN_EDEVICE, which
 * dgen_synchronize reports, and leaves every buffer index in bounds.
 * DGEN_TUNE_SEPARATE_EXPERTS (0 or 1): 1 runs the bf16 expert gate-up and
 * down GEMMs as two launches instead of one persistent launch (measurement;
 * FP8 experts always use two, with the activation quantization between).
 * DGEN_TUNE_STATIC_ITEMS (0 or 1): 1 makes the one-launch expert GEMMs take
 * their items in a fixed stride (CTA b: items b, b + grid, ...) instead of
 * claiming the next untaken item from a counter (measurement).
 * DGEN_TUNE_PAIRS (0, 1 or 2): which dense GEMMs run on CTA pairs
 * (tcgen05.mma.cta_group::2 over 256-row tiles) instead of one-CTA 128-row
 * tiles: 0 (automatic) the LM head and the self-conditioning p0_hat E, whose
 * long K streams make the pair's halved per-SM intake pay; 1 none; 2 also the
 * QKV and O projections, whose short K (2816 and 4096 over 256 rows) measured
 * slower on pairs, the cluster's start-up and end costing more than the
 * intake saves (measurement).  DGEN_TUNE_CHUNK_ORDER (0, 1 or 2): the order
 * of the routed experts' token chunks, which is the order in which the expert
 * GEMMs take their items (no result depends on it): 0 (automatic) largest
 * expert first where the two expert GEMMs run as two launches (E4M3 experts,
 * DGEN_TUNE_SEPARATE_EXPERTS), expert id order for the one persistent launch;
 * 1 id order; 2 largest expert first (measurement). */
#define DGEN_TUNE_EXPERT_CHUNK 0
#define DGEN_TUNE_ATTN_SPLITS 1
#define DGEN_TUNE_ROUTER_SPLITS 2
#define DGEN_TUNE_QKV_SPLITS 3
#define DGEN_TUNE_ATTN_KERNEL 4
#define DGEN_TUNE_ROUTE_BARRIER_EXTRA 5
#define DGEN_TUNE_SEPARATE_EXPERTS 6
#define DGEN_TUNE_STATIC_ITEMS 7
#define DGEN_TUNE_PAIRS 8
#define DGEN_TUNE_CHUNK_ORDER 9
int dgen_set_tuning(dgen_handle* h, int32_t key, int32_t value);

/* Test hook (teacher forcing of the routing): while set, every layer of the
 * prompt pass (prompt_ids_dev [L][B*P][k]) and/or of the decoder pass
 * (canvas_ids_dev [L][B*C][k]) uses the given expert ids instead of its own
 * top-k; the gates are still the softmax of the layer's own router logits over
 * the given ids.  Ids are clamped to [0, E).  NULL releases a pass.  Used to
 * compare the arithmetic of all rows with a reference whose routing differs
 * at near-ties. */
int dgen_force_routing(dgen_handle* h, const int32_t* prompt_ids_dev, const int32_t* canvas_ids_dev);

/* Number of experts each layer routed at least one token to in the last
 * decoder or prompt pass (their weights are what the expert GEMMs read):
 * touched_host[n_layers], host memory.  Synchronizes the stream. */
int dgen_expert_usage(dgen_handle* h, int32_t* touched_host);

/* Execution flags (default 0).  DGEN_FLAG_NO_GRAPH: run every decoder pass as
 * individual launches instead of replaying a captured CUDA graph.
 * DGEN_FLAG_NO_PDL: launch kernels without programmatic dependent launch
 * (this one is process-wide).  For debugging and measurement. */
#define DGEN_FLAG_NO_GRAPH 1u
#define DGEN_FLAG_NO_PDL 2u
int dgen_set_flags(dgen_handle* h, uint32_t flags);

/* Diagnostic capture of the routing decisions of subsequent decoder passes
 * (dgen_denoise_step): for every layer l, the top-k expert ids [rows][k]
 * (int32, in rank order) are copied to ids_dev + l*rows*k and, if logits_dev
 * is not NULL, the fp32 router logits [rows][E] to logits_dev + l*rows*E,
 * rows = B*C.  Either pointer may be NULL; both NULL stops the capture.  Used
 * to count routing flips against a reference (the router's top-k over
 * near-equal logits is discontinuous). */
int dgen_capture_routing(dgen_handle* h, int32_t* ids_dev, float* logits_dev);

/* Diagnostic capture of the residual stream of subsequent decoder passes
 * (dgen_denoise_step): after layer l (attention and MoE blocks, residual adds
 * included) the fp32 residual h [rows][d] is copied to h_dev + l*rows*d, rows =
 * B*C.  NULL stops the capture.  Used to compare each layer with a reference
 * given the same input (layer-wise teacher forcing). */
int dgen_capture_residual(dgen_handle* h, float* h_dev);

/* Diagnostic read-out of internal buffers after the last call (for tests):
 * which = 0 residual stream h [rows][d] fp32; 1 normed activations [rows][d]
 * bf16; 2 rotated queries [B][Hq][n_q][hd] bf16; 3 attention output
 * [rows][Hq*hd] bf16; 4 / 5 the K / V cache of layer `layer`
 * [B][Hkv][prompt_max + C][hd] bf16; 6 / 7 the per-position argmax (int32) /
 * confidence or entropy (fp32) [B*C] of the last sampler call (layer is then
 * ignored but must be valid); 8 the gated expert activations [rows*k][w] bf16
 * (permuted rows); with expert_fp8 also 9 / 10 their E4M3 bytes [rows*k][w] and
 * row scales [rows*k] fp32, 11 / 12 the gathered E4M3 token rows [rows*k][d]
 * and their scales; 13 the token of each permuted row [rows*k] int32, 14 the
 * gated down-projection output of each permuted row [rows*k][d] fp32, 15 the
 * gate of each permuted row [rows*k] fp32; with a shared FFN 16 its gated
 * activations [rows][ws] bf16 and 21 its slice outputs [ceil(ws/w)][rows][d]
 * fp32, with expert_fp8 also 17 / 18 their E4M3 bytes [rows][ceil(ws/w) wp]
 * (each w-wide slice padded with zeros to wp = w rounded up to 128) and row
 * scales, 19 / 20 the E4M3 token rows in natural order [rows][d] and their
 * scales; with self-conditioning, after a decoder pass, 22 p0_hat [B*C][V]
 * bf16, 23 K-split partial number `layer` of u = p0_hat E [B*C][d] fp32, 24
 * the normed u [B*C][d] bf16, 25 the FFW activations [B*C][w_sc] bf16 and 26
 * K-split partial number `layer` of the state z [B*C][d] fp32 (u and z are the
 * sums of their partials in index order; for 23 and 26 `layer` past the last
 * partial gives EINVAL) (EINVAL where the buffer does not exist).  rows and n_q are those of the last
 * pass (B*C and C after a decoder pass).  Copies min(bytes, buffer size)
 * bytes to dst_dev.  Buffers are reused across layers: after a pass they hold
 * the last layer's values. */
int dgen_debug_read(dgen_handle* h, int32_t which, int32_t layer, void* dst_dev, uint64_t bytes);

/* Kernel classes for dgen_set_timing / dgen_get_timing. */
#define DGEN_K_QKV 0            /* QKV projection GEMM (+RoPE, cache write) */
#define DGEN_K_ATTENTION 1      /* attention (+ split combine) */
#define DGEN_K_OPROJ 2          /* output projection GEMM (K-split partials) */
#define DGEN_K_ROUTER 3         /* router GEMM and the routing launch (top-k, permutation, gather) */
#define DGEN_K_EXPERT_GATE_UP 4 /* grouped expert gate-up GEMM (+GELU * up), shared FFN included */
#define DGEN_K_EXPERT_DOWN 5    /* grouped expert down GEMM (* gate), shared FFN included */
#define DGEN_K_SHARED_FFN 6     /* unused: the shared FFN runs inside the grouped expert launches */
#define DGEN_K_LM_HEAD 7        /* LM head GEMM (+softmax statistics; the final norm is fused into the last combine) */
#define DGEN_K_SAMPLER 8        /* statistics merge + sampler */
#define DGEN_K_OTHER 9          /* embedding + first norm, residual add + norm, expert combine + norm */
#define DGEN_K_SELF_COND 10     /* self-conditioning: p0_hat, p0_hat E, norm, FFW */
#define DGEN_K_CLASSES 11

/* Per-kernel-class device time, measured with CUDA events recorded on the
 * handle's stream around each launch of the classes whose bit is set in
 * class_mask (0 disables).  For measurement only; adds two event records per
 * timed launch. */
int dgen_set_timing(dgen_handle* h, uint32_t class_mask);

/* Waits for the stream, then returns the summed device time (ms) and the
 * number of timed launches of class cls since the last call for that class,
 * and resets them. */
int dgen_get_timing(dgen_handle* h, int32_t cls, double* total_ms, int64_t* launches);

const char* dgen_status_str(int status);

/* Allocation-free sampler step, for callers that must not allocate device
 * memory: code on a latency-critical serving path, where cudaMalloc/cudaFree
 * would synchronise the whole device and stall the other streams; hosts and
 * frameworks that own all device memory through their own allocator and do
 * not let a plug-in library allocate; deployments with a device-memory budget
 * fixed in advance.  (The pages have no counterpart: this is an interface
 * choice of this library.)
 *
 * Does what dgen_set_logits followed by dgen_sample_commit do, without a
 * handle: reads fp32 logits [batch][canvas][vocab], updates tok_dev and
 * committed_dev [batch][canvas] in place (argmax commit of the most confident
 * uncommitted positions, Philox re-noise of the rest, at step s of T), and
 * writes the confidences to conf_dev_or_null [batch][canvas] if not NULL.
 * stream: a cudaStream_t (NULL = legacy default stream); asynchronous.
 *
 * Scratch: one fixed array in the library's device memory of
 * 262144 * 12 + 8192 * 8 + 256 bytes (about 3.1 MB), present on every GPU that
 * loads the library until the process exits.  Limits: batch * canvas <= 8192
 * and batch * canvas * (vocab / 256) <= 262144 (e.g. 256 rows at vocab
 * 262144, 2048 rows at vocab 32768); canvas <= 1024; vocab a multiple of 256.
 * Larger sizes return DGEN_ESCRATCH and enqueue nothing.  It calls no
 * cudaMalloc, cudaFree or other allocating routine.
 *
 * Every call uses the same scratch array, which keeps the previous call's
 * contents (each call writes every scratch value before reading it): calls
 * that can overlap on the GPU (other streams, other threads) race and must be
 * ordered by the caller.  The first call on a device looks up the array's
 * device address (cudaGetSymbolAddress, once per device, under a lock) and
 * keeps it for the life of the process; make that first call before any stream
 * capture.  A device reset (cudaDeviceReset, or a reset of the primary context)
 * after the first call is not supported: the kept address would be stale. */
int dgen_sample_from_logits_noalloc(const float* logits_dev, int32_t* tok_dev, uint8_t* committed_dev,
                                    int32_t batch, int32_t canvas, int32_t vocab, int32_t s, int32_t T,
                                    uint64_t seed, float tau_max, float tau_min, int32_t commit_per_step,
                                    float* conf_dev_or_null, void* stream);

/* Diagnostic entry point (exercised by the tests): the same product with E4M3
 * operands (OCP FP8, one byte per element, row-major [M][K] and [N][K]) through
 * the GEMM core's tcgen05 kind::f8f6f4 path, D fp32 [M][N].  K a multiple of 16.
 * Errors: EINVAL, ECUDA. */
int dgen_gemm_e4m3(const void* a_dev, const void* b_dev, float* d_dev, int32_t M, int32_t N, int32_t K,
                   void* stream);

/* Diagnostic entry point (exercised by the tests): D[M][N] (fp32, row-major,
 * ldd = N) = A[M][K] * B[N][K]^T with A, B bf16 row-major device arrays,
 * through the same tcgen05 tensor-core GEMM core the decoder uses.  K a
 * multiple of 8; stream as in dgen_create.  Errors: EINVAL, ECUDA. */
int dgen_gemm_bf16(const void* a_dev, const void* b_dev, float* d_dev, int32_t M, int32_t N, int32_t K,
                   void* stream);

/* Diagnostic entry point (exercised by the tests): the same product on CTA
 * pairs (a cluster of two CTAs computes each 256 x 256 tile with
 * tcgen05.mma.cta_group::2, each CTA holding half of the A rows and half of
 * the B rows; the form the decoder's LM head uses).
 * Same arguments and errors as dgen_gemm_bf16. */
int dgen_gemm_bf16_pair(const void* a_dev, const void* b_dev, float* d_dev, int32_t M, int32_t N, int32_t K,
                   void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DGEN_H */
