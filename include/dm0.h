/*
 * dm0.h - C ABI of the DM0 dual-expert merged-attention path on NVIDIA B200
 * (sm_100a): inference (prefix pass, Euler loop), with an FP8 E4M3 VLM MLP
 * option, the DM0.5 time-modulated action expert as a configuration, and one
 * flow-matching training step of the action expert.
 *
 * What it computes (page title and section of the sources):
 *   - DM0 architecture notes (dregs-remover.com/news/27019), section 1: in each
 *     of L Qwen3-style layers a VLM branch (hidden Hv) and an action-expert
 *     branch (hidden Ha) make their own Q/K/V with the same head count and
 *     head_dim; the two sets are concatenated along the sequence axis, run
 *     through one attention, split back, and each branch applies its own
 *     O-projection, residual and SwiGLU MLP.  DM0-base: L = 28, Hv = 2048,
 *     Ha = 1024, 16 query heads, 8 KV heads, head_dim 128, action dim 32,
 *     chunk 50.
 *   - "DM0.5: High-Performance Embodied VLA and OpenDM Open Source
 *     Introduction", section 5.1 (the prefix runs once and its per-layer KV
 *     cache is kept), 5.2 (action_in_proj -> action expert -> action_out_proj
 *     gives the velocity v(x_t, t | c)), 5.3 (Euler integration from noise
 *     x_1 with diffusion_steps = 10 returns the whole chunk; training regresses
 *     v onto u_t = eps - a at x_t = t eps + (1 - t) a under an action mask),
 *     6.3 (FP8 E4M3 for the prefix MLP's GEMMs), 6.5 (fixed shapes and a
 *     graph captured once and replayed); section 5.2 also names the time MLP
 *     and per-layer time modulators of the DM0.5 action expert.
 *
 * Conventions shared by every entry point:
 *   - Every call returns a dm0_status; no call throws or aborts.  After a
 *     failure dm0_last_error() describes it.
 *   - "device pointer" arguments are CUDA device addresses of the current
 *     device, owned by the caller, and must stay valid until the work queued on
 *     `stream` has finished.  `stream` is a cudaStream_t (NULL = legacy default
 *     stream).  Device-pointer calls are asynchronous on `stream`.
 *   - Layouts are dense row-major with the innermost index last.  bf16 is the
 *     IEEE-754 bfloat16 bit pattern in a uint16_t.
 *   - Kernels never trap.  A kernel that meets an internal timeout or a bad
 *     index sets a device error word and returns early; the next call on the
 *     context (or dm0_sync) reports DM0_EDEVICE and the context stays in
 *     that state until dm0_clear_error().
 *   - A context is bound to the CUDA device that was current at dm0_create and
 *     is not thread-safe: calls on one context must be serialised by the caller.
 */
#ifndef DM0_H_
#define DM0_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct dm0_ctx dm0_ctx;

/* Model shapes and capacity.  Constraints checked by dm0_create:
 *   head_dim in {32, 64, 128}; n_q % n_kv == 0;
 *   hidden_v, hidden_a, n_q*head_dim, n_kv*head_dim multiples of 32 and
 *   hidden_v, hidden_a, inter_v, inter_a, n_q*head_dim multiples of 128
 *   (tensor-core tile rows), 2*inter multiples of 128;
 *   action_dim <= 64; chunk >= 1; max_batch >= 1; max_prefix >= 1;
 *   max_prefix + chunk <= 65536; time_mod in {0, 1}. */
typedef struct {
  int layers;       /* decoder layers per branch (28 for DM0-base) */
  int hidden_v;     /* VLM hidden size (2048) */
  int inter_v;      /* VLM SwiGLU intermediate size (6144) */
  int hidden_a;     /* action-expert hidden size (1024) */
  int inter_a;      /* action-expert SwiGLU intermediate size (3072) */
  int n_q;          /* query heads (16) */
  int n_kv;         /* key/value heads (8) */
  int head_dim;     /* 128 */
  int chunk;        /* action tokens per sample S (50) */
  int action_dim;   /* A (32) */
  int max_batch;    /* largest B any call will use */
  int max_prefix;   /* largest P any call will use */
  float rope_theta; /* 1e6 */
  float rms_eps;    /* 1e-6 */
  int time_mod;     /* 0: DM0 action expert (time embedding added to the input);
                       1: DM0.5 time-modulated action expert (DM0.5 page, section 5.2):
                       a time MLP turns tau(t) into a condition c, and every
                       action-expert RMSNorm (attention, MLP, final) becomes
                       x / rms(x) * (1 + scale) + shift with [scale | shift | gate] =
                       W_m silu(c) + b_m, the gate scaling the sublayer's residual
                       add; the static gains of those norms are unused.  The blob
                       gains the time tensors (see dm0_load_weights); the Euler loop
                       runs as per-layer kernels. */
} dm0_config;

typedef enum {
  DM0_OK = 0,
  DM0_EINVAL = -1,   /* null pointer or malformed argument */
  DM0_ESHAPE = -2,   /* B, P, steps or a size outside the context's capacity */
  DM0_ENOMEM = -3,   /* device or host allocation failed */
  DM0_ECUDA = -4,    /* a CUDA runtime/driver call failed */
  DM0_EDEVICE = -5,  /* a kernel reported an internal timeout or bad index */
  DM0_ESTATE = -6    /* call out of order (no weights, or no KV cache yet) */
} dm0_status;

/* Allocate a context on the current CUDA device: weight storage, the
 * per-layer KV cache for max_batch x max_prefix, activation buffers and the
 * RoPE table (built on the device).  *out receives the context.  Nothing is
 * allocated afterwards except CUDA-graph instantiations (one per distinct
 * (B, P, steps) of dm0_denoise).
 * Environment switches read here (scheduling only: none changes what is
 * computed, and every one keeps its default when unset):
 *   DM0_NO_PDL=1         no programmatic dependent launch between kernels
 *   DM0_NO_GRAPH=1       batched Euler loops as direct launches, no CUDA graph
 *   DM0_NO_PERSIST=1     one observation's Euler loop as per-layer kernels
 *   DM0_PERSIST_SPLITS=n attention key splits per KV head of that loop (7)
 *   DM0_PERSIST_FASTBAR=0  its grid barriers with full fences (see dm0_denoise)
 *   DM0_RASTER_BAND=n    persistent-GEMM tile bands of n m-tiles (default: n-fastest
 *                        for weights up to 64 MB, 64-m-tile bands above)
 *   DM0_QKV_EPI=8        the QKV GEMM epilogue on eight warps instead of four
 *   DM0_PERSIST_TRACE=1, DM0_GEMM_TRACE=1  timestamp buffers (dm0_debug_view) */
dm0_status dm0_create(const dm0_config* cfg, dm0_ctx** out);

/* Weight blob size in bytes for `cfg`. */
size_t dm0_weights_bytes(const dm0_config* cfg);

/* Copy weights from a HOST blob (caller keeps ownership) into the context,
 * repacking for the kernels (Q/K/V rows fused, gate/up rows interleaved in
 * 64-row blocks).  Synchronous.  Blob layout, all little-endian, no padding:
 *   for branch in (VLM, action expert): for l in 0..layers-1:
 *     attn_norm f32[H] | Wq bf16[n_q*D][H] | Wk bf16[n_kv*D][H] |
 *     Wv bf16[n_kv*D][H] | q_norm f32[D] | k_norm f32[D] |
 *     Wo bf16[H][n_q*D] | mlp_norm f32[H] | Wg bf16[I][H] | Wu bf16[I][H] |
 *     Wd bf16[H][I]
 *   then W_in bf16[Ha][A] | b_in f32[Ha] | final_norm f32[Ha] |
 *        W_out bf16[A][Ha] | b_out f32[A]
 *   and, when time_mod = 1: W_ti bf16[Ha][Ha] | b_ti f32[Ha] | W_to bf16[Ha][Ha] |
 *        b_to f32[Ha] | W_mf bf16[2Ha][Ha] | b_mf f32[2Ha] (time_mlp_in, time_mlp_out,
 *        the final norm's [scale | shift] modulator), then for l in 0..layers-1:
 *        W_ma bf16[3Ha][Ha] | b_ma f32[3Ha] | W_mm bf16[3Ha][Ha] | b_mm f32[3Ha]
 *        (the attention and MLP pre-norms' [scale | shift | gate] modulators)
 * Matrices are [out][in].  `bytes` must equal dm0_weights_bytes(). */
dm0_status dm0_load_weights(dm0_ctx* ctx, const void* blob, size_t bytes);

/* Prefix pass (DM0.5 page, section 5.1): runs the VLM branch alone over the
 * prefix and fills the context-owned KV cache.
 *   prefix_emb: device bf16 [B][P][hidden_v] prefix embeddings.
 * The cache holds, per layer, K after QK-norm and RoPE (positions 0..P-1) and
 * V, as two planes of bf16 [layers][B][n_kv][P][head_dim] (see dm0_kv_view).
 * Returns DM0_ESHAPE unless 1 <= B <= max_batch and 1 <= P <= max_prefix. */
dm0_status dm0_prefill(dm0_ctx* ctx, const void* prefix_emb, int B, int P, void* stream);

/* Shape buckets: make dm0_denoise for (B, P, steps) ready ahead of time, so a
 * later call of that shape does no capture.  Where the Euler loop runs as
 * per-layer kernels (B >= 2, or the persistent kernel unavailable) this
 * captures and caches its CUDA graph without launching anything; the
 * single-observation persistent loop takes B, P and steps as launch arguments
 * and needs nothing.  The KV cache and its committed shape are untouched.
 * Call it outside any stream capture (it captures on the context's own
 * stream).  Returns DM0_ESTATE without weights, DM0_ESHAPE outside the
 * context's capacity or unless 1 <= steps <= 1000. */
dm0_status dm0_prepare(dm0_ctx* ctx, int B, int P, int steps);

/* Device pointers of the KV-cache planes (context-owned, valid until
 * dm0_destroy).  With the (B, P) of the last prefill or dm0_kv_commit, plane
 * element [l][b][h][p][d] sits at index (((l*B + b)*n_kv + h)*P + p)*head_dim + d.
 * Capacity: layers*max_batch*n_kv*max_prefix*head_dim elements per plane. */
dm0_status dm0_kv_view(dm0_ctx* ctx, void** k_plane, void** v_plane);

/* Declare that the caller wrote a KV cache of shape (B, P) through
 * dm0_kv_view (for a denoise over an externally provided prefix cache). */
dm0_status dm0_kv_commit(dm0_ctx* ctx, int B, int P);

/* Flow-matching Euler sampler (DM0.5 page, sections 5.2-5.3) over the cached
 * prefix of the last prefill / kv_commit: x = noise;
 * for k in 0..steps-1: t = 1 - k/steps, x <- x - v(x, t)/steps.
 *   noise:      device f32 [B][chunk][action_dim] (x_1), read once.
 *   actions:    device f32 [B][chunk][action_dim] output x_0 (may alias noise).
 *   velocities: device f32 [steps][B][chunk][action_dim] per-step v, or NULL.
 * One observation (B = 1) with head_dim 128 runs the whole loop as ONE
 * persistent kernel (one CTA per SM, grid barriers between the phases of a
 * layer; DM0_PERSIST_SPLITS at dm0_create sets its attention key splits per
 * KV head, default 7; each barrier arrival is one release reduction and the
 * wait an acquire spin, with no full fences around them, unless
 * DM0_PERSIST_FASTBAR=0 was set, which adds them); otherwise, when the kernel cannot be resident on every
 * SM, and when the environment variable DM0_NO_PERSIST=1 was set at
 * dm0_create, the loop is a chain of per-layer kernels captured once per
 * (B, P, steps) as a CUDA graph and replayed (launched directly when
 * velocities are requested).  No host work happens inside the loop.  The
 * persistent loop's split-K sums arrive in any order, so repeated calls are
 * not bitwise identical.
 * With time_mod = 1 each call first builds, for its K steps, every norm's
 * [1 + scale | shift | gate] from the time MLP and the modulators, and the two
 * shifts of each layer projected through its QKV and gate/up weights (one pass
 * over those weights per call); the layers then run the per-layer kernels with
 * the per-step gains, a feature bias after the pending 1/rms and a gate on each
 * residual add (the persistent loop covers the DM0 expert only).
 * Returns DM0_ESTATE without a cache, DM0_ESHAPE unless 1 <= steps <= 1000. */
dm0_status dm0_denoise(dm0_ctx* ctx, const float* noise, int steps, float* actions, float* velocities,
                       void* stream);

/* Observation -> action chunk from HOST memory: copies prefix_emb (host bf16
 * [B][P][hidden_v]) and noise (host f32 [B][chunk][action_dim]) to the device,
 * runs dm0_prefill and dm0_denoise, copies the chunk back to `actions` (host
 * f32) and waits for `stream`.  Host buffers should be pinned for full copy
 * bandwidth; pageable memory works but is slower. */
dm0_status dm0_infer_host(dm0_ctx* ctx, const void* prefix_emb, const float* noise, int B, int P, int steps,
                          float* actions, void* stream);

/* One dual-expert layer `layer` with both branches over the concatenated
 * [prefix; suffix] sequence (DM0 architecture notes, section 1), for tests:
 *   h_prefix  device f32 [B][P][hidden_v]   VLM residual stream in
 *   h_suffix  device f32 [B][chunk][hidden_a] action residual stream in
 *   out_prefix/out_suffix: device f32, same shapes, residual streams out
 *   k_out/v_out: device bf16 [B][n_kv][P][head_dim], the prefix K (after
 *   QK-norm + RoPE) and V of this layer.
 * Prefix rows attend to prefix keys only; suffix rows to all P + chunk keys.
 * Uses the context's buffers; overwrites the KV cache slot of `layer`.  The
 * layer has no flow time, so a time_mod context returns DM0_EINVAL. */
dm0_status dm0_merged_layer(dm0_ctx* ctx, int layer, const float* h_prefix, const float* h_suffix, int B, int P,
                            float* out_prefix, float* out_suffix, void* k_out, void* v_out, void* stream);

/* Flow-matching training step (DM0.5 page, section 5.3). ------------------ */

/* Floats of the gradient buffer of dm0_train_step for `cfg`: per action layer
 * attn_norm[Ha] | Wq[n_q*D][Ha] | Wk[n_kv*D][Ha] | Wv[n_kv*D][Ha] | q_norm[D] |
 * k_norm[D] | Wo[Ha][n_q*D] | mlp_norm[Ha] | Wg[Ia][Ha] | Wu[Ia][Ha] | Wd[Ha][Ia],
 * then W_in[Ha][A] | b_in[Ha] | final_norm[Ha] | W_out[A][Ha] | b_out[A]: the
 * action-expert part of the weight blob, in fp32, no padding. */
size_t dm0_grad_floats(const dm0_config* cfg);

/* One training step of the DM0 action expert over the context's prefix cache
 * (the last dm0_prefill or dm0_kv_commit; its B samples):
 *   x_t = t eps + (1 - t) a and u = eps - a per sample; v = the expert's velocity
 *   at (x_t, t); loss = sum over valid entries of (v - u)^2 / their count (0 if
 *   none); grads = dloss / d(every action-expert and head parameter).
 *   a, eps:  device f32 [B][chunk][action_dim]; t: device f32 [B];
 *   mask:    device u8 [B][chunk][action_dim], nonzero = valid entry;
 *   loss:    device f32 [1], written;
 *   grads:   device f32 [dm0_grad_floats(cfg)] (16-byte aligned), written;
 *   kv_grads: null (knowledge insulation: the prefix K/V is a constant), or
 *            device f32 [2][layers][B][n_kv][P][head_dim]: dloss/dK then dloss/dV
 *            of the cache (where the gradient would enter the VLM).
 * Forward projections and every dX = dY W, dW = dY^T X run on the tensor-core
 * GEMM with bf16 operands and fp32 accumulation; the first call after
 * dm0_load_weights builds transposed copies of the action weights (0.9 GB at
 * DM0-base widths) and the step's buffers.  Asynchronous on `stream`.
 * Returns DM0_ESTATE without weights or cache, DM0_EINVAL for null pointers,
 * misaligned grads or a time_mod context, DM0_ESHAPE if chunk * head_dim > 8192. */
dm0_status dm0_train_step(dm0_ctx* ctx, const float* a, const float* eps, const float* t, const uint8_t* mask,
                          float* loss, float* grads, float* kv_grads, void* stream);

/* Kernel-level entry points used by the unit tests. -------------------- */

/* Tensor-core GEMM in fp32 accumulation:
 *   swap == 0: C[M][N]  = A[M][K] * B[N][K]^T, C written.
 *   swap == 1: C[N][M] += A[M][K] * B[N][K]^T transposed (A plays the weight
 *              operand, B the token operand, N <= 128); C must be zeroed by
 *              the caller; `splits` K-splits accumulate atomically.
 * A, B device bf16 K-contiguous; C device f32.  M % 128 == 0 when swap == 1;
 * K % 64 == 0 and K >= 64; splits >= 1 (only 1 when swap == 0). */
dm0_status dm0_op_gemm(dm0_ctx* ctx, const void* A, const void* B, float* C, int M, int N, int K, int swap,
                       int splits, void* stream);

/* Per-row FP8 E4M3 quantisation on the GPU (the operand step of the FP8
 * prefix MLP, DM0.5 page, section 6.3).  Row r of x, y[c] = x[r][c], times
 * gain[c] when gain is not null, times 1/sqrt(ssq[r] / cols + eps_rms) when ssq
 * is not null (a pending RMSNorm; eps from the context's config), in fp32:
 *   scales[r] = max_c |y[c]| / 448 (an fp32 division; 1 for an all-zero row),
 *   codes[r][c] = E4M3(y[c] / scales[r]), the quotient an IEEE fp32 division
 *   and the conversion round-to-nearest-even, saturating at +-448.
 * x device [rows][cols], fp32 when x_f32 != 0 else bf16 (16-byte aligned);
 * gain device f32 [cols] (16-byte aligned) or null; ssq device f32 [rows] or
 * null; codes device u8 [rows][cols] (8-byte aligned; OCP E4M3 bit patterns);
 * scales device f32 [rows].  rows >= 1, cols >= 8 and cols % 8 == 0, else
 * DM0_ESHAPE; null required pointers or misalignment give DM0_EINVAL.
 * Asynchronous on `stream`. */
dm0_status dm0_op_quant_e4m3(dm0_ctx* ctx, const void* x, int x_f32, int rows, int cols, const float* gain,
                             const float* ssq, void* codes, float* scales, void* stream);

/* FP8 E4M3 tensor-core GEMM with per-row scales on both operands:
 *   C[m][n] = sa[m] * sb[n] * sum_k e4m3(A[m][k]) e4m3(B[n][k]),
 * products of codes accumulated in fp32.  A device u8 [M][K] and B device u8
 * [N][K] codes, K-contiguous (16-byte aligned); sa device f32 [M]; sb device
 * f32 [N] (16-byte aligned); C device f32 [M][N], written.  M >= 1, N % 128 ==
 * 0, K % 128 == 0, else DM0_ESHAPE.  Asynchronous on `stream`. */
dm0_status dm0_op_gemm_e4m3(dm0_ctx* ctx, const void* A, const float* sa, const void* B, const float* sb, float* C,
                            int M, int N, int K, void* stream);

/* Merged GQA attention of one segment pair, for tests:
 *   q:  device bf16 [B][Tq][n_q][head_dim]
 *   ka/va: device bf16 [B][n_kv][Ta][head_dim]; kb/vb: [B][n_kv][Tb][head_dim]
 *   (kb/vb may be NULL with Tb = 0)
 *   o:  device bf16 [B][Tq][n_q][head_dim]
 * Every query row sees all Ta + Tb keys; scale 1/sqrt(head_dim); query head h
 * reads KV head h / (n_q / n_kv).  splits >= 1 splits the keys (64-key
 * blocks) across CTAs and combines partial softmax states. */
dm0_status dm0_op_attention(dm0_ctx* ctx, const void* q, const void* ka, const void* va, int Ta, const void* kb,
                            const void* vb, int Tb, void* o, int B, int Tq, int splits, void* stream);

/* Device pointer of an internal activation buffer, for tests that check
 * intermediate results.  `name` is one of: h_v, xn_v, q_v, o_v, act_v, ssq_v
 * (VLM side, rows = B*P tokens) and h_a, xn_a, q_a, o_a, act_a, ssq_a, x,
 * k_s, v_s (action side, rows = B*chunk tokens).  Layouts: h_* f32 [rows][H];
 * xn_* bf16 [rows][H] (gain * h of the pending RMSNorm); q_*, o_* bf16
 * [rows][n_q*head_dim]; act_* bf16 [rows][inter]; ssq_* f32 [2][H/64][rows]
 * (the attention norm's, then the MLP norm's sums of squares of h, one partial
 * sum per 64-column group, which the consumer adds in group order); x f32 [rows][action_dim];
 * k_s/v_s bf16 [B][n_kv][chunk][head_dim].  Context-owned; contents are only
 * meaningful after the call that fills them has completed.
 * "loop_trace" (NULL unless DM0_PERSIST_TRACE=1 was set at dm0_create): u64
 * marks of the persistent Euler loop (runs of <= 16 steps), [phase][CTA][16]:
 * %globaltimer at 0 phase start, 1 operand staged, 2 first accumulator (or S
 * tile) ready, 3 results issued, 4 release fence done, 5 barrier arrival, 6 MMA
 * warp saw the operand, 7 MMA warp issued its last MMA, 8 operand copies issued
 * (inside the preceding barrier), 9 copies landed; attention items: 10 / 12 S
 * of key block 0 / 1 read, 11 / 13 its P written, 14 O read out, 15 first PV
 * issued; GEMM phases, SM cycles (clock64): 12 phase start, 13 copies' issue
 * entered, 15 copies issued, 11 copies landed, 14 first pair's operand built,
 * 10 staging done;
 * phase 0 is the input of step 0, then per step 5 phases per layer (QKV,
 * attention, O, gate/up, down) and the step boundary.
 * "gemm_trace" (NULL unless DM0_GEMM_TRACE=1 was set at dm0_create): u64
 * %globaltimer marks of the last 64 persistent-GEMM launches (round robin, in
 * launch order), [launch][CTA (num_sms rows)][16] = entry, setup done, past the
 * dependency wait, first k-block landed, first tile's MMAs issued, first
 * accumulator complete, first tile's epilogue done, last tile's epilogue done
 * (0 for one-tile CTAs), last TMA copy issued, exit; QKV launches: slots 10-13
 * SM cycles (clock64) of the first epilogue thread's last tile (first 128-column
 * group entered, its first head's RMS pass done, that head's RoPE pass done,
 * second group done); CTA 0's slots 14 and 15 hold (M << 32 | N) and
 * (K << 32 | tile width); rows of CTAs that did not run in a launch keep stale
 * values.
 * "tm_mod", "tm_bqkv", "tm_bgu" (time_mod contexts, NULL before the first
 * dm0_denoise or dm0_prepare): the modulation tables of the last Euler loop of
 * K steps, f32 [K][(6*layers + 2)*hidden_a] (per layer [attention: 1 + scale |
 * shift | gate][MLP: 1 + scale | shift | gate], then the final norm's
 * [1 + scale | shift]), [layers][K][(n_q + 2 n_kv) head_dim] and
 * [layers][K][2 inter_a] (the shifts through the QKV and interleaved gate/up
 * weights). */
dm0_status dm0_debug_view(dm0_ctx* ctx, const char* name, void** ptr);

/* Merged GQA attention that allocates nothing, for callers that cannot call
 * cudaMalloc: a real-time control loop that must not allocate once it runs,
 * code that runs inside stream capture, or a host whose device memory is
 * owned by another allocator.  It needs no dm0_ctx (creating one allocates).
 * The pages have no counterpart: this is a deployment variant of
 * dm0_op_attention.
 *
 * Same arguments, layouts and result as dm0_op_attention, with the head
 * layout given explicitly (n_q, n_kv, head_dim in {32, 64, 128}).  When the
 * keys are split (splits > 1, after clamping to the number of 64-key blocks),
 * the partial softmax states go to a fixed device-side scratch area inside
 * the library (about 2 MB, held by every GPU that loads the library until the
 * process exits) of 32 slots: B * n_kv * ceil((n_q/n_kv) * Tq / 128) * splits
 * must be <= 32, otherwise DM0_ESHAPE.  The caller passes inputs and outputs only.
 *
 * The first call on a device looks up the scratch's device address and sets
 * the kernels' shared-memory limit; make that first call before any stream
 * capture.  Every call shares the one scratch area and resets its counters
 * on `stream`: calls that overlap on the GPU (different streams without
 * ordering) race and give wrong results.  Asynchronous on `stream`; returns
 * DM0_EINVAL / DM0_ESHAPE / DM0_ECUDA on bad arguments or launch failure. */
dm0_status dm0_attention_noalloc(const void* q, const void* ka, const void* va, int Ta, const void* kb,
                                 const void* vb, int Tb, void* o, int B, int Tq, int n_q, int n_kv, int head_dim,
                                 int splits, void* stream);

/* FP8 E4M3 prefix MLP (DM0.5 page, section 6.3). ---------------------------- */

/* enable != 0: from now on every VLM-branch MLP of this context (dm0_prefill
 * and the VLM half of dm0_merged_layer) runs its gate/up and down GEMMs in
 * FP8 E4M3: the weights are quantised once here, per output channel, from the
 * resident bf16 weights (and again by every later dm0_load_weights); each
 * GEMM's operand is quantised per token from fp32 just before it (the gate/up
 * operand is the normalised residual rms(h) * g, the down operand the SwiGLU
 * output; the rules of dm0_op_quant_e4m3); products accumulate in fp32 and
 * both scales are applied in the GEMM's epilogue.  The action expert stays bf16.  enable == 0 returns
 * to the bf16 MLP (the FP8 copies are kept).
 * Needs loaded weights (DM0_ESTATE) and hidden_v, inter_v multiples of 128
 * (DM0_ESHAPE).  The first enable allocates the FP8 weights (1 byte per MLP
 * weight of the VLM) and operands (max_batch * max_prefix * (hidden_v +
 * 5 inter_v) bytes: codes and the fp32 SwiGLU output); DM0_ENOMEM if that
 * fails.  The weight quantisation is
 * queued on `stream`. */
dm0_status dm0_set_prefix_fp8(dm0_ctx* ctx, int enable, void* stream);

/* FP8 packing (host). ---------------------------------------------------- */

/* Packs a row-major fp32 matrix into FP8 E4M3 codes with one scale per row,
 * the weight format of an FP8 GEMM whose rows are output channels (DM0.5 page,
 * section 6.3: FP8 E4M3 for the prefix MLP's gate/up/down GEMMs, with scales).
 * Per row r: s_r = max_k |x[r][k]| / 448 (1 for an all-zero row); code[r][k] is
 * the E4M3 value nearest x[r][k] / s_r (1 sign, 4 exponent bits with bias 7, 3
 * mantissa bits, no infinities, largest finite 448; ties to even; values beyond
 * +-448 saturate), so x[r][k] ~= s_r * e4m3(code[r][k]).  Scales and quotients
 * are computed in double.
 *   x:      host f32 [rows][cols], read only.
 *   codes:  host u8 [rows][cols] (OCP E4M3 bit patterns; no NaN is produced).
 *   scales: host f32 [rows].
 * Host-only and synchronous; no GPU is needed.  Returns DM0_EINVAL for null
 * pointers or a non-finite input, DM0_ESHAPE unless rows, cols >= 1. */
dm0_status dm0_pack_e4m3_rows(const float* x, int64_t rows, int64_t cols, uint8_t* codes, float* scales);

/* Instrumentation. ------------------------------------------------------- */

/* Number of kernels this context has enqueued so far (a replayed graph counts
 * every kernel it contains).  Host-side counter; never synchronises. */
uint64_t dm0_launch_count(const dm0_ctx* ctx);

/* Kernel sites dm0_probe can time. */
enum {
  DM0_SITE_VLM_QKV = 0,     /* prefix pass: Q/K/V GEMM (+QK-norm, RoPE, cache write) */
  DM0_SITE_VLM_ATTN = 1,    /* prefix pass: attention */
  DM0_SITE_VLM_O = 2,       /* prefix pass: O GEMM (+residual) */
  DM0_SITE_VLM_GATEUP = 3,  /* prefix pass: gate/up GEMM (+SwiGLU) */
  DM0_SITE_VLM_DOWN = 4,    /* prefix pass: down GEMM (+residual) */
  DM0_SITE_ACT_QKV = 5,     /* Euler loop: the same five action-expert kernels */
  DM0_SITE_ACT_ATTN = 6,
  DM0_SITE_ACT_O = 7,
  DM0_SITE_ACT_GATEUP = 8,
  DM0_SITE_ACT_DOWN = 9,
  DM0_SITE_STEP = 10,       /* Euler step boundary (velocity, update, next input) */
  DM0_SITE_LOOP = 11,       /* the whole Euler loop as one persistent kernel (one observation; the
                               per-layer sites 5-10 are then not launched) */
  DM0_SITE_COUNT = 12
};

/* Time the launches of the sites in `site_mask` (bit i = site i) with CUDA
 * events recorded on the launching stream around each launch; 0 turns the
 * probe off.  Enabling resets the record.  A timed launch follows an event
 * record, so it runs in plain stream order instead of overlapping the
 * previous kernel, and while any site is probed dm0_denoise launches its
 * kernels directly instead of replaying its graph.  Events are created on
 * demand (256 at a time, at most 16384). */
dm0_status dm0_probe(dm0_ctx* ctx, int site_mask);

/* Wait for the recorded events of `site` and return its number of timed
 * launches and their summed duration in milliseconds. */
dm0_status dm0_probe_read(dm0_ctx* ctx, int site, int* launches, double* total_ms);

/* Failure-path self-test (no counterpart on the pages): launches a kernel
 * whose bounded mbarrier wait — the same wait every pipeline of the library
 * uses — is given an mbarrier nothing ever arrives on.  The wait gives up
 * after `limit_us` microseconds (1..1e6), the kernel sets the device error
 * word and returns; dm0_sync then reports DM0_EDEVICE and dm0_clear_error
 * makes the context usable again.  Asynchronous on `stream`. */
dm0_status dm0_selftest_timeout(dm0_ctx* ctx, int limit_us, void* stream);

/* Errors and lifetime. -------------------------------------------------- */

/* Wait for `stream`, then report DM0_EDEVICE if a kernel raised the device
 * error word, else DM0_OK (DM0_ECUDA if the wait itself failed). */
dm0_status dm0_sync(dm0_ctx* ctx, void* stream);

/* Device error word (0 when clean; bit 0..4: producer / MMA / epilogue
 * timeout, bad index, drain timeout). */
int dm0_device_error(const dm0_ctx* ctx);

/* Clear the device error word and re-zero the split-K accumulators and
 * counters so the context can be used again.  Synchronous. */
dm0_status dm0_clear_error(dm0_ctx* ctx);

/* Human-readable description of the last failure on `ctx` (never NULL). */
const char* dm0_last_error(const dm0_ctx* ctx);

/* Free everything the context owns.  NULL is ignored. */
void dm0_destroy(dm0_ctx* ctx);

#ifdef __cplusplus
}
#endif
#endif /* DM0_H_ */
