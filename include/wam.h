/*
 * wam.h -- C ABI of the B200 (sm_100a) MoT world-action-model forward.
 *
 * What is computed.  A Mixture-of-Transformers world-action model has a
 * video expert and an action expert, each a stack of N DiT blocks; block i
 * of the action expert attends over the concatenation [K^v_i; K^a_i],
 * [V^v_i; V^a_i] of the video expert's block-i keys/values and its own, so
 * the video expert runs once per chunk and publishes z = {(K^v_i, V^v_i)}
 * (RealtimeWAM summary page, section 前置知识: "Mixture-of-Transformers",
 * "KV 缓存").  The action chunk is then integrated by Euler flow matching,
 * a_{t_{j-1}} = a_{t_j} - (t_j - t_{j-1}) v(a_{t_j}, t_j), whose one-step form
 * from t is the endpoint f = a_t - t v (section 前置知识, "流匹配与速度场去噪").
 * The two experts overlap as the Cross-Expert Wavefront Pipeline: video
 * stream P^v_i -> record(e_i) -> Attn^v_i -> R^v_i, action stream P^a_i ->
 * wait(e_i) -> Attn^a_i -> R^a_i (sections 核心方法 and 方法步骤详情; the
 * tokendh.com article, CEWP section).  The joint one-step variant adds the SNR
 * time shift, the consistency endpoints and an unmerged LoRA on the action
 * expert (Flash-WAM close reading, sections 概念 / 方法 / 数据与训练流程).
 *
 * Conventions of every entry point.
 *   - Pointers named dev_* are device pointers on the context's device; the
 *     caller owns them and keeps them alive until the enqueued work finishes.
 *     Pointers named host_* are host pointers (pageable or pinned).
 *   - Streams are cudaStream_t values passed as void* (NULL = legacy default
 *     stream).  All calls only enqueue work and return; synchronise on the
 *     stream named in each call's comment.
 *   - Layouts are row-major, C-contiguous, fp32 unless stated.
 *   - Errors: argument errors return WAM_ERR_INVALID_ARG before anything is
 *     enqueued; CUDA errors return WAM_ERR_CUDA (text: wam_last_error); a
 *     device-side bounded wait that gave up is reported as WAM_ERR_TIMEOUT by
 *     wam_check_device_status.  No call aborts the process.
 *   - One context per host thread; a context is bound to the device that was
 *     current at wam_init.
 */
#ifndef MOT_DIT_B200_WAM_H
#define MOT_DIT_B200_WAM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  WAM_OK = 0,
  WAM_ERR_INVALID_ARG = 1,
  WAM_ERR_UNSUPPORTED = 2,
  WAM_ERR_OOM = 3,
  WAM_ERR_CUDA = 4,
  WAM_ERR_TIMEOUT = 5,
  WAM_ERR_STATE = 6
} wam_status;

typedef enum { WAM_FP32 = 0, WAM_BF16 = 1 } wam_dtype;
typedef enum { WAM_SCHED_SEQUENTIAL = 0, WAM_SCHED_CEWP = 1 } wam_sched;

/* Model shapes.  N blocks per expert; widths d_video / d_action; n_heads x
 * head_dim attention (A = n_heads * head_dim, shared by both experts); FFN
 * widths; l_cond + l_video video-expert tokens (L_v) and l_action action
 * tokens of dimension action_dim per sample; batch samples.
 * video_patch_dim > 0 selects patch-vector video input (joint variant).
 * lora_rank > 0 adds an unmerged LoRA (scale lora_scale) to the action
 * expert's QKV / out / FFN projections.  video_has_output: the video expert's
 * last block and output map run (joint variant).  dtype: WAM_BF16 (bf16
 * weights and GEMM operands, fp32 accumulation and residual stream, head_dim
 * 64) or WAM_FP32 (fp32 everywhere, debug precision).  wam_init rejects
 * (WAM_ERR_INVALID_ARG) shapes its kernels do not cover: expert widths above
 * 1536; on the bf16 path widths that are not multiples of 64 (128 for
 * ffn_video and the attention width), more than 64 action tokens per sample
 * or 256 per chunk, and a LoRA rank that is not a multiple of 64. */
typedef struct {
  int n_blocks, d_video, d_action, n_heads, head_dim, ffn_video, ffn_action;
  int l_cond, l_video, l_action, action_dim, video_patch_dim;
  int batch, lora_rank;
  float lora_scale;
  int video_has_output;
  int dtype;
} wam_config;

typedef struct wam_ctx wam_ctx;

/* Fill *out with synthetic preset k (1: tiny fp32; 2: Fast-WAM-shaped bf16,
 * 28 blocks, 1536/768 widths, 64+1024 video tokens, 32 action tokens;
 * 3: as 2 (the 10-step teacher schedule is chosen per call); 4: as 2 with
 * batch 8 and 2048 video tokens; 5: joint one-step, 30 blocks at 1536,
 * 1024 patch tokens of dim 192, 16 action tokens, LoRA rank 128).
 * Returns WAM_ERR_INVALID_ARG for an unknown k. */
wam_status wam_preset(int k, wam_config* out);

/* Create a context on the current device: generates the seeded parameters
 * on the device (parameter p, element e: SplitMix64 counters
 * (seed XOR p*0x9E3779B97F4A7C15) + 2e + {0,1}, Box-Muller, N(0, 0.02) for
 * weights / biases / modulation tables / LoRA factors, 1 for norm gains;
 * rounded to bf16 for bf16 models), allocates the K/V cache, the
 * activations and the workspaces, and creates the per-block events.
 * Synchronous.  *out is set only on WAM_OK.  WAM_ERR_OOM when a device
 * allocation fails, or would take the context past the byte budget given in
 * the environment variable WAM_DEVICE_MEMORY_LIMIT (unset or 0: no budget);
 * everything allocated so far is released. */
wam_status wam_init(const wam_config* cfg, uint64_t seed, wam_ctx** out);

/* Release everything the context owns (device memory, events, graphs).
 * Synchronises the device first.  NULL is a no-op. */
void wam_destroy(wam_ctx* ctx);

/* Video expert of one chunk on `stream`: x = [cond; video] per sample, N DiT
 * blocks at timestep t_video; block i publishes K^v_i / V^v_i into the cache
 * and records its ready event right after its projection.  The last block's
 * attention and remainder run only when the model has a video output.
 * dev_video: [B, l_video, d_video]; dev_cond: [B, l_cond, d_video] (NULL iff
 * l_cond == 0).  Before overwriting block i's K/V it waits for the previous
 * chunk's action attention of block i. */
wam_status wam_video_forward(wam_ctx* ctx, const float* dev_video, const float* dev_cond, float t_video,
                             void* stream);

/* One Euler step of the action expert on `stream`, in place on
 * dev_actions [B, l_action, action_dim]: a <- a - (t_from - t_to) v(a, t_from).
 * Block i waits for the video expert's block-i event before its attention.
 * Requires a wam_video_forward on this context first (else WAM_ERR_STATE).
 * t_from > t_to, both in [0, 1], else WAM_ERR_INVALID_ARG. */
wam_status wam_action_step(wam_ctx* ctx, float* dev_actions, float t_from, float t_to, void* stream);

/* Whole chunk: video expert once (at t = 0) and S Euler steps from the noise
 * dev_noise [B, l_action, action_dim] along host_t_sched (S + 1 values,
 * t_S = first > ... > t_0 = last, within [0, 1]; NULL = uniform j/S), result
 * in dev_actions_out.  mode: WAM_SCHED_CEWP runs the experts on stream_video
 * and stream_action with one event per block (action attention i waits only
 * for video block i); WAM_SCHED_SEQUENTIAL runs everything on stream_video.
 * Both produce bitwise-identical results.  use_graph: capture the chunk once
 * per (S, mode) into a CUDA graph and replay it (pointers and the schedule
 * are read from device memory, so later calls may change them).  The work
 * starts after all work previously enqueued on both streams and completes on
 * stream_video.  1 <= S <= 64. */
wam_status wam_infer_chunk(wam_ctx* ctx, const float* dev_video, const float* dev_cond, const float* dev_noise,
                           float* dev_actions_out, int S, const float* host_t_sched, int mode, int use_graph,
                           void* stream_video, void* stream_action);

/* Same as wam_infer_chunk with host buffers: copies host_video / host_cond /
 * host_noise into context-owned device buffers on stream_video, runs the
 * chunk, copies the actions back into host_actions_out and synchronises
 * stream_video before returning. */
wam_status wam_infer_chunk_host(wam_ctx* ctx, const float* host_video, const float* host_cond,
                                const float* host_noise, float* host_actions_out, int S, const float* host_t_sched,
                                int mode, int use_graph, void* stream_video, void* stream_action);

/* Joint one-step variant (1 video step, 1 action step): sigma_v / sigma_a
 * from the unshifted levels u_video / u_action by sigma = s u / (1 + (s-1) u);
 * x_sigma = (1 - sigma_v) x_0 + sigma_v eps_v, a_sigma = (1 - sigma_a) a_0 +
 * sigma_a eps_a; outputs the action endpoint f^a = a_sigma - sigma_a v^a and
 * the video endpoint f^v = c_skip x_sigma + c_out (x_sigma - sigma_v v^v),
 * c_skip = sd^2/(sigma^2+sd^2), c_out = sigma sd / sqrt(sigma^2+sd^2),
 * sd = 0.5.  Requires video_patch_dim > 0 and video_has_output.
 * dev_video_clean / dev_video_eps: [B, l_video, video_patch_dim];
 * dev_action_clean / dev_action_eps: [B, l_action, action_dim];
 * outputs of the same shapes.  Streams, mode and use_graph as in
 * wam_infer_chunk. */
wam_status wam_joint_one_step(wam_ctx* ctx, const float* dev_video_clean, const float* dev_video_eps,
                              const float* dev_action_clean, const float* dev_action_eps, float u_video,
                              float u_action, float shift_video, float shift_action, float* dev_video_out,
                              float* dev_action_out, int mode, int use_graph, void* stream_video,
                              void* stream_action);

/* Chunk with a multi-step video expert (RealtimeWAM summary page, 未来方向
 * (2): the wavefront carried over to a video expert that keeps several
 * denoising steps).  Requires video_patch_dim > 0 and video_has_output.
 * The video latents start from dev_video_eps (level 1) and take n_video
 * flow-matching Euler steps x <- x - (s_j - s_{j-1}) v^v(x, s_j) along
 * host_sched_video (n_video + 1 levels falling from 1 to the last, within
 * [0, 1]; NULL = uniform j / n_video), each a full forward of the video
 * expert; the result x_0 goes to dev_video_out [B, l_video, video_patch_dim].
 * The action expert then takes S Euler steps from dev_noise along
 * host_t_sched (as in wam_infer_chunk) over the K/V of the LAST video forward:
 * under WAM_SCHED_CEWP only that forward records the per-block events, and
 * action block i's attention waits for video block i of it.  mode, use_graph
 * and the streams as in wam_infer_chunk; 1 <= n_video, S <= 64. */
wam_status wam_infer_chunk_multistep(wam_ctx* ctx, const float* dev_video_eps, const float* dev_noise,
                                     float* dev_video_out, float* dev_actions_out, int n_video,
                                     const float* host_sched_video, int S, const float* host_t_sched, int mode,
                                     int use_graph, void* stream_video, void* stream_action);

/* TACD target forward (Teacher-Anchored Consistency Distillation, forward
 * only: the targets one training step of the action expert's LoRA is fitted
 * to; RealtimeWAM summary page, sections 前置知识 "一致性蒸馏", 核心方法 and
 * 方法步骤详情).  On `stream`, with device buffers:
 *   a_t = (1 - t) a_clean + t eps;
 *   the video expert once (t_v = 0) on dev_video / dev_cond, its K/V shared
 *   by all three networks;
 *   the frozen teacher -- the student's base weights, LoRA off -- runs K
 *   Euler steps from (a_t, t) over the uniform grid t_k = t k / K down to 0:
 *   a_0^T, and its first state a~_s at s = t (K - 1) / K;
 *   the student (the LoRA model `student`) gives the endpoint
 *   f(a_t, t) = a_t - t v, so v_student = (a_t - f) / t;
 *   the EMA target (the LoRA model `ema`; it may be `student` itself) gives
 *   f^-(a~_s, s) (for s = 0 the endpoint map is the identity);
 *   u_TA = (a_t - a_0^T) / t, u_CD = (a_t - f^-) / t;
 *   losses[0] = L_TA = E||v_student - u_TA||^2, losses[1] = L_CD =
 *   E||v_student - u_CD||^2 (squared L2 over one sample's [l_action,
 *   action_dim], mean over the batch), losses[2] = L_CD + lambda L_TA.
 * dev_action_clean, dev_eps and the optional outputs dev_u_ta, dev_v_student,
 * dev_u_cd, dev_a_t, dev_a0_teacher are [B, l_action, action_dim]; losses is
 * 3 floats (required).  student and ema: contexts of the same config with
 * lora_rank > 0 on one device; the EMA's K/V cache is overwritten with the
 * student's.  0 < t <= 1, 1 <= K <= 64, else WAM_ERR_INVALID_ARG.  Buffers
 * for the intermediate states are allocated in `student` on first use. */
wam_status wam_tacd_targets(wam_ctx* student, wam_ctx* ema, const float* dev_video, const float* dev_cond,
                            const float* dev_action_clean, const float* dev_eps, float t, int K, float lambda,
                            float* dev_u_ta, float* dev_v_student, float* dev_u_cd, float* dev_losses,
                            float* dev_a_t, float* dev_a0_teacher, void* stream);

/* Copy every parameter, in generation order, as fp32 into host_buf (matrix
 * padding removed).  With host_buf == NULL only *nbytes is set.  Synchronous.
 * WAM_ERR_INVALID_ARG if *nbytes is too small. */
wam_status wam_export_params(wam_ctx* ctx, float* host_buf, size_t* nbytes);

/* Overwrite every parameter from host_buf (same order and size as
 * wam_export_params; values are rounded to bf16 for bf16 models).  Synchronous. */
wam_status wam_import_params(wam_ctx* ctx, const float* host_buf, size_t nbytes);

/* Copy block `block`'s K (which = 0) or V (which = 1) cache, [B, H,
 * l_cond + l_video + l_action, head_dim], as fp32 into host_buf (size
 * checked against *nbytes; NULL: report size).  Synchronous. */
wam_status wam_read_kv(wam_ctx* ctx, int block, int which, float* host_buf, size_t* nbytes);

/* Synchronise the context's device and report device-side failures of the
 * bounded waits (WAM_ERR_TIMEOUT, then clears the flag) or CUDA errors. */
wam_status wam_check_device_status(wam_ctx* ctx);

/* Pixel front-end of the patch-input (joint) model: the Flash-WAM setting
 * cuts 128 x 128 RGB frames into 16 x 16 patches of 3 x 8 x 8 = 192 values
 * (Flash-WAM close reading, 数据与训练流程).  inverse = 0: dev_frames
 * [B, F, C, H, W] (channel-first) -> dev_patches [B, F (H/p)(W/p), C p p];
 * token f (H/p)(W/p) + py (W/p) + px, feature c p^2 + iy p + ix holds pixel
 * (f, c, py p + iy, px p + ix).  inverse = 1: the other way (dev_patches read,
 * dev_frames written), e.g. for the video endpoint.  H and W multiples of p.
 * Enqueued on `stream`.  (The pages name a VAE encoder in the end-to-end
 * latency but give no architecture or weights: none is built.) */
wam_status wam_patchify(const float* dev_frames, float* dev_patches, int B, int F, int C, int H, int W, int p,
                        int inverse, void* stream);

/* Failure-path test hook (tests only; every context of the process on the
 * current device).  With extra > 0, the last piece of a split GEMM tile that
 * is its CTA's final segment waits for `extra` more partial tiles than exist,
 * giving up after limit_ns nanoseconds: the bounded wait runs out on a count
 * nothing raises, the CTA winds down (its copies and MMAs drained, TMEM
 * released), and wam_check_device_status then reports WAM_ERR_TIMEOUT and
 * clears the tickets, so the next call is clean.  extra = 0 restores the
 * normal wait (2 s limit, never reached).  Synchronous; call it outside
 * stream capture.  No GPU fault is involved. */
wam_status wam_test_peer_wait(int extra, unsigned long long limit_ns);

/* Number of kernel launches one chunk enqueues for (S, mode) (graph or not). */
int wam_chunk_kernel_count(wam_ctx* ctx, int S);

/* Kernel classes of wam_profile_chunk. */
typedef enum {
  WAM_PROF_VIDEO_NORM = 0, WAM_PROF_VIDEO_QKV, WAM_PROF_VIDEO_ATTN, WAM_PROF_VIDEO_OPROJ,
  WAM_PROF_VIDEO_FFN_UP, WAM_PROF_VIDEO_FFN_DOWN, WAM_PROF_VIDEO_TEMB, WAM_PROF_VIDEO_IO,
  WAM_PROF_ACTION_NORM, WAM_PROF_ACTION_QKV, WAM_PROF_ACTION_ATTN, WAM_PROF_ACTION_OPROJ,
  WAM_PROF_ACTION_FFN_UP, WAM_PROF_ACTION_FFN_DOWN, WAM_PROF_ACTION_TEMB, WAM_PROF_ACTION_IO,
  WAM_PROF_ACTION_BLOCK, /* persistent action-block launches (attention + R_i + next P_i, one per block) */
  WAM_PROF_CLASSES
} wam_prof_class;

/* Measurement: run one chunk (S uniform steps) with the sequential schedule
 * on `stream` -- captured once into a CUDA graph with an event-record node
 * before and after every launch, then replayed -- and
 * return per class the summed launch durations host_ms[WAM_PROF_CLASSES] and
 * the launch counts host_counts[WAM_PROF_CLASSES].  Synchronises `stream`.
 * Arguments as in wam_infer_chunk.  (QKV and the action in / out projections
 * count the whole projection; the fp32 path's QK-norm kernel is part of QKV.) */
wam_status wam_profile_chunk(wam_ctx* ctx, const float* dev_video, const float* dev_cond, const float* dev_noise,
                             float* dev_actions_out, int S, void* stream, float* host_ms, int* host_counts);

/* Kinds of wam_trace_chunk records. */
typedef enum {
  WAM_TRACE_START = 0,        /* chunk start (video stream) */
  WAM_TRACE_VIDEO_KV = 1,     /* video block i's projection done: K^v_i / V^v_i published, e_i recorded */
  WAM_TRACE_VIDEO_END = 2,    /* video block i's remainder done */
  WAM_TRACE_ACTION_ATTN = 3,  /* action stream reaches Attn^a_i (after its wait on e_i) */
  WAM_TRACE_ACTION_END = 4,   /* action block i done (its remainder, and the next block's projection on the
                                 persistent path) */
  WAM_TRACE_END = 5           /* chunk end (video stream, after the join) */
} wam_trace_kind;

/* Measurement of the wavefront: the chunk (S uniform steps, `mode`) captured
 * into a CUDA graph with a timing event at every block boundary of both
 * streams (the event nodes replace the dependent-launch overlap at those
 * points), replayed once to warm up and once timed.  Writes up to `capacity`
 * records of 4 floats (kind, block, Euler step, ms since the start record)
 * into host_ms and the number of records into *count.  Synchronises
 * stream_video.  Arguments otherwise as in wam_infer_chunk. */
wam_status wam_trace_chunk(wam_ctx* ctx, const float* dev_video, const float* dev_cond, const float* dev_noise,
                           float* dev_actions_out, int S, int mode, void* stream_video, void* stream_action,
                           float* host_ms, int capacity, int* count);

const char* wam_status_str(wam_status s);
const char* wam_last_error(wam_ctx* ctx);

/* ---- single-operation entry points (tests and measurement) ------------ */

/* C[M, N] = X[M, K] W[N, K]^T + bias (fp32 out), X / W bf16 (dtype WAM_BF16)
 * on the tcgen05 path or fp32 (WAM_FP32) on the SIMT path.  swap selects
 * the few-token orientation (weight on the 128-row MMA operand, M <= 256).
 * The bf16 path splits the k-blocks of all output tiles evenly over its
 * persistent CTAs (stream-K; partial tiles summed in k order): `splits` is
 * the number of CTAs per output tile when swapped, else the number of CTAs
 * (0: one per SM).  K must be a multiple of 64, ld of X / W equal K, and N a
 * multiple of 32 unless swapped, on the bf16 path.  Uses a private workspace
 * (allocated on first use or growth); enqueued on `stream`. */
wam_status wam_op_linear(int dtype, const void* dev_x, const void* dev_w, const float* dev_bias, float* dev_out,
                         int M, int N, int K, int swap, int splits, void* stream);

/* The same product through the video expert's tile shapes (bf16 only, normal
 * orientation, fp32 out): bn = 128, 192 or 256 output features per CTA tile.
 * mode 0: single CTAs.  mode 1 (bn 256): CTA pairs -- two CTAs of a cluster
 * share each M = 256 tensor-core MMA (the 2-SM form), each holding its own
 * 128 rows of X and half of the 256 rows of W.  mode 2: single-CTA tiles
 * launched as clusters of two CTAs; a tile whose k-range the stream-K split
 * gives to the two CTAs of one cluster is finished in column halves, each
 * CTA's half-partial of the other's columns crossing in shared memory.
 * ctas = persistent CTAs (0: one per SM; even for mode 2, rounded down to
 * pairs for mode 1).  K a multiple of 64, N a multiple of 32.
 * mode 3: the swapped orientation of the action expert (M <= 64 token rows
 * as the MMA's N operand, bn ignored), each 128-feature tile split over
 * ctas = 2..8 CTAs of one cluster, one equal k-range each (K / 64 a multiple
 * of ctas, and 32 (M <= 32) or 64 a multiple of 4 ctas); the pieces are summed
 * in rank (= k) order in shared memory, each CTA finishing its share of the
 * token columns.  Returns WAM_ERR_INVALID_ARG for other shapes or values. */
wam_status wam_op_linear_tiled(const void* dev_x, const void* dev_w, const float* dev_bias, float* dev_out, int M,
                               int N, int K, int bn, int mode, int ctas, void* stream);

/* out[B*Lq, H*Dh] = softmax(q k^T / sqrt(Dh)) v per (sample, head) over
 * cache rows [0, Lk); q [B, H, Lq, Dh], k / v [B, H, Lcache, Dh]; bf16
 * (Dh = 64, split-KV when splits > 1) or fp32.  Enqueued on `stream`. */
wam_status wam_op_attention(int dtype, const void* dev_q, const void* dev_k, const void* dev_v, void* dev_out,
                            int B, int H, int Dh, int Lq, int Lk, int Lcache, int splits, void* stream);

/* The joint action attention of the chunk path: out[B*Lq, H*64] (bf16) =
 * softmax(q k^T / 8) v per (sample, head) over cache rows [0, Lk), the
 * action queries against the concatenated [K^v_i; K^a_i] (RealtimeWAM
 * summary page, 前置知识 "Mixture-of-Transformers" / "KV 缓存").  q bf16
 * [B, H, Lq, 64] with Lq <= 64; k / v bf16 [B, H, Lcache, 64].  The keys of
 * each (sample, head) are split over `splits` CTAs of a cluster (1, 2, 4 or
 * 8 with splits * Lq <= 279; 0 chooses from the SM count) whose partials
 * are merged in split order,
 * so the result does not depend on timing.  Cache rows below `ready` are
 * read before the kernel waits for the previous kernel on the stream, so they
 * must be complete when the call is enqueued (0: no such assumption).
 * WAM_ERR_INVALID_ARG for other shapes; enqueued on `stream`. */
wam_status wam_op_attention_joint(const void* dev_q, const void* dev_k, const void* dev_v, void* dev_out, int B, int H,
                                  int Lq, int Lk, int Lcache, int ready, int splits, void* stream);

/* h[M, d] = rms(x) * (dev_gain ? gain : 1 + scale) + (dev_shift ? shift : 0)
 * per row, rms(x) = x / sqrt(mean(x^2) + 1e-6): the RMSNorm / AdaLN
 * modulation prologue of every block (and, with a gain, the final norm).
 * x fp32 [M, d]; h bf16 (dtype WAM_BF16) or fp32 (WAM_FP32); d a multiple
 * of 4 and <= 1536; scale / shift / gain fp32 [d] (dev_scale required when
 * dev_gain is NULL).  Enqueued on `stream`. */
wam_status wam_op_norm_mod(int dtype, const float* dev_x, void* dev_h, int M, int d, const float* dev_scale,
                           const float* dev_shift, const float* dev_gain, void* stream);

/* Allocation-free split-KV attention.  (An addition for deployment; the
 * paper has no counterpart.)  Same computation, kernel and arguments as
 * wam_op_attention with dtype WAM_BF16, Dh = 64 and splits >= 2, for callers
 * that cannot let a library allocate device memory while they run -- a
 * control loop that must not call cudaMalloc after start-up (the call can
 * synchronise the device and has unbounded latency), or a process whose
 * device memory budget belongs to another allocator.  Its scratch (per-split
 * partial outputs, row maxima and sums, and the tickets that pick the
 * combining CTA) is a fixed 8 MiB + 4 KiB array compiled into the library,
 * held by every GPU that loads the library until the process exits; the call
 * makes no allocation.
 *   - Limits: B * H * s * (64*64 + 128) floats <= 2^21 and B * H <= 1024,
 *     where s is the number of non-empty key splits (at most 32);
 *     1 <= Lq <= 64.  A call beyond them returns WAM_ERR_UNSUPPORTED and
 *     enqueues nothing.
 *   - The first call on a device looks up the array's device address and
 *     sets the kernel's shared-memory limit (once per device, with that
 *     device current); make that first call before any stream capture.
 *     Both are kept for the life of the process: after a cudaDeviceReset
 *     that device's cached address is stale, so do not call this entry point
 *     again on a device that has been reset.
 *   - Every call shares the array: calls that overlap on the GPU (other
 *     streams, other threads) race.  Each call clears the tickets it uses
 *     before its kernel runs.
 *   - Enqueued on `stream`; returns WAM_ERR_INVALID_ARG for bad arguments. */
wam_status wam_op_attention_noalloc(const void* dev_q, const void* dev_k, const void* dev_v, void* dev_out, int B,
                                    int H, int Lq, int Lk, int Lcache, int splits, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOT_DIT_B200_WAM_H */
