// Internal launcher interface of the MoT world-action-model kernels.
// Host code (the C ABI, the schedules) calls only these functions; each one
// enqueues kernels on the given stream and returns the launch error code.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace wam {

// Launch with programmatic stream serialization (dependent launch) when
// enabled (default on; WAM_PDL=0 in the environment turns it off at load).
bool pdl_enabled();
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                     Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Widest row the RMSNorm / modulation kernels and the GEMM norm prologue take.
constexpr int kRowNormMax = 1536;

constexpr int kMaxSteps = 64;  // Euler steps per chunk held in the device schedule

// Per-call inputs read by the first/last kernels of a chunk.  They live in
// device memory so a captured CUDA graph reads the current call's pointers and
// timestep schedule instead of baked-in values.
struct VideoIo {
  const float* video;   // [B, L_vid, d_v] (or patch vectors [B, L_vid, P_v])
  const float* cond;    // [B, L_c, d_v] or null
  const float* eps;     // joint variant: video noise [B, L_vid, P_v]
  float* video_out;     // joint variant: video endpoint [B, L_vid, P_v]
  float t;              // video timestep (noise level) of the chunk
  float u;              // joint variant: unshifted level; shift applied on device
  float shift;          // joint variant: SNR shift s_v (0: use t as is)
  float vsched[65];     // multi-step video: noise levels s_{N_v} > ... > s_0 of the video Euler steps
  int vsteps;           // multi-step video: N_v (0: one pass)
};
struct ActionIo {
  const float* a_in;    // chunk start [B, L_a, P_a] (noise, or the caller's state)
  const float* a_clean; // joint variant: clean action to noise
  float* a_out;         // result [B, L_a, P_a]
  float sched[kMaxSteps + 1];  // t_S, ..., t_0
  int steps;
  float u;              // joint variant: unshifted action level
  float shift;          // joint variant: SNR shift s_a (0: not the joint variant)
};

enum Epi : int {
  kEpiStoreF32 = 0,  // out_f32[m, n] = acc + bias[n]
  kEpiGateRes = 1,   // out_f32[m, n] += gate[n] * (acc + bias[n])
  kEpiGelu = 2,      // out_act[m, n] = gelu_tanh(acc + bias[n])
  kEpiQkv = 3,       // bias, per-head QK-RMSNorm with gains, RoPE, scatter to Q and the KV cache
  kEpiEuler = 4,     // a[m, n] -= (t_j - t_{j-1}) * (acc + bias[n]); also writes the next in-proj input
  kEpiVideoOut = 5,  // joint variant: video endpoint f^v = c_skip x + c_out (x - sigma v)
  kEpiScaleAct = 6,  // out_act[m, n] = scale * (acc + bias[n]) (act dtype): the LoRA down-projection s x A^T
  kEpiVideoEuler = 7,  // multi-step video: x[m, n] -= (s_j - s_{j-1}) (acc + bias[n]) into out_f32 (the latents),
                       // also the next in-projection input out_act (ld a_next_ld) and, after the last step,
                       // the chunk's video vio->video_out
};

struct EpiArgs {
  int kind = 0;
  float scale = 1.f;  // kEpiScaleAct
  const float* bias = nullptr;
  const float* gate = nullptr;
  float* out_f32 = nullptr;
  void* out_act = nullptr;
  int ld_out = 0;
  // QKV scatter
  const float* gq = nullptr;
  const float* gk = nullptr;
  const float* rope_cos = nullptr;  // [cache_len][Dh/2]
  const float* rope_sin = nullptr;
  void* q_out = nullptr;            // [B, H, seq_len, Dh]
  void* k_cache = nullptr;          // [B, H, cache_len, Dh] (block base)
  void* v_cache = nullptr;
  int seq_len = 0, cache_len = 0, cache_off = 0, n_heads = 0, head_dim = 0, attn_dim = 0;
  // Euler / endpoints
  const ActionIo* aio = nullptr;
  const VideoIo* vio = nullptr;
  int step = 0;
  void* a_next = nullptr;           // next in-proj input (act dtype), ld = a_next_ld
  int a_next_ld = 0;
  const float* x_sigma = nullptr;   // joint variant: noised video patches
  // Output tensor maps of the normal orientation's TMA-store epilogues
  // (box 32 rows): map_o = the output matrix (fp32 [M, N], box 32 cols; bf16
  // [M, N], box 64 cols) or Q ([B*H][L][64]); map_o2 = the K/V cache
  // ([2*N*B*H][L_v + L_a][64]).  zq0 / zk0 / zv0: matrix index of (b=0, h=0).
  const CUtensorMap* map_o = nullptr;
  const CUtensorMap* map_o2 = nullptr;
  int zq0 = 0, zk0 = 0, zv0 = 0;
  // Swapped orientation only: the B operand (tokens x K) is computed in the
  // kernel as rms(nb_x) * (nb_gain or 1 + nb_scale) + nb_shift from fp32 rows
  // nb_x [tokens][K] (ld = K) instead of being loaded; map_b is then unused.
  const float* nb_x = nullptr;
  const float* nb_scale = nullptr;
  const float* nb_shift = nullptr;
  const float* nb_gain = nullptr;
  // Normal orientation only: the launch first writes its own A operand,
  // na_h[r] = rms(na_x[r]) * (1 + na_scale) + na_shift as bf16 for every
  // token row r (fp32 rows, ld = K; na_h is the memory map_a reads).  Rows
  // are taken one at a time from na_cnt[0] by whichever CTAs run, counted
  // done in na_cnt[1]; A tiles are loaded once all rows are done; the last
  // CTA out (na_cnt[2]) sets the three counters back to zero.  The counters
  // are private to one stream's launches.
  const float* na_x = nullptr;
  const float* na_scale = nullptr;
  const float* na_shift = nullptr;
  void* na_h = nullptr;
  int* na_cnt = nullptr;
};

// C[m, n] = sum_k X[m, k] W[n, k] (+ epilogue), bf16 operands via TMA into
// tcgen05 tiles.  `swap`: the weight is the 128-row MMA operand (features on
// TMEM lanes) and the tokens are the N operand -- used when there are few tokens.
struct TcGemm {
  const CUtensorMap* map_a;  // A operand: [rows_a, K] (3-D: z = matrix index)
  const CUtensorMap* map_b;  // B operand: [rows_b, K]
  int rows_a, rows_b, K;
  int z_a, z_b;              // matrix index (block) of each operand
  int bn;                    // N tile (32, 64, 128, 256)
  int splits;                // swapped: CTAs = tiles * splits (each tile's K split evenly)
  bool swap;
  int max_ctas;              // normal: persistent grid size (0: one CTA per SM)
  bool pair;                 // normal, bn 256: CTA pairs share M = 256 MMAs (2-SM tensor-core tiles);
                             // the B map's box is then bn / 2 rows (each CTA loads half)
  bool csplit;               // normal, single CTAs: launch as clusters of two (even grid); a tile whose
                             // k-range stream-K splits between the two CTAs of a cluster is finished
                             // in column halves, the partials crossing in shared memory
  int cred;                  // swapped, splits > 1: launch as clusters of `splits` CTAs (<= 8, dividing
                             // the k-blocks and bn / 4) when cred == splits; each tile's pieces are then
                             // summed in shared memory, each CTA finishing bn / splits token columns
  float* ws;                 // partial tiles: 2 * CTAs * 128 * bn floats (tc_gemm_ws_floats)
  int* tickets;              // two per output tile, zero on entry, left zero
  unsigned* status;
};

// Workspace floats the launch needs for K-split partial tiles.
size_t tc_gemm_ws_floats(const TcGemm& g);
// Ticket ints the launch needs (two per 128-row output tile).
size_t tc_gemm_tickets(const TcGemm& g);
// CTA pairs the device holds at once (0 before prepare_tc_gemm).
int tc_gemm_max_pairs();
// Partial tiles the last piece of a split tile can bring into its operand
// ring at once (the fast reduction path); tiles split into more pieces are
// summed from global memory instead.  Normal orientation: the smallest ring
// of the 128- / 256-wide instances.
int tc_gemm_ring_partials(int bn, bool swap, bool fused_norm);

cudaError_t launch_tc_gemm(const TcGemm& g, const EpiArgs& e, cudaStream_t s);
// Failure-path test hook of the split-tile wait (0, kWaitLimitNs: off).
cudaError_t set_peer_wait_test(int extra, unsigned long long limit_ns);
// Sets the kernels' shared-memory attributes; call once per device before any
// launch (and never during stream capture).
cudaError_t prepare_tc_gemm();

// fp32 SIMT GEMM (debug precision): C = X W^T + epilogue; X [M, K] with row
// stride ldx, W [N, K] (row stride K).
cudaError_t launch_f32_gemm(const float* X, int ldx, const float* W, int M, int N, int K, const EpiArgs& e,
                            cudaStream_t s);

// fp32 path: per-head QK-RMSNorm + RoPE + scatter of a raw projection [M, 3A].
cudaError_t launch_qkv_post_f32(const float* qkv, int M, const EpiArgs& e, cudaStream_t s);

// h[m, :] = rms(x[m, :]) * (gain ? gain : 1 + scale) + (shift ? shift : 0);
// h rows ldh apart (0: d).
cudaError_t launch_norm_mod(const float* x, void* h, bool h_bf16, int M, int d, const float* scale,
                            const float* shift, const float* gain, cudaStream_t s, int ldh = 0);

// Timestep conditioning of one expert: tau(t) -> c -> m, then mod[i] = m + T_i
// for every block.  t = io_t[0] (device scalar); weights in `bf16` or fp32.
struct TembArgs {
  const float* t;       // device scalar
  const void* w1; const float* b1;   // [d, 256]
  const void* w2; const float* b2;   // [d, d]
  const void* wm; const float* bm;   // [6d, d]
  const float* T0; size_t T_stride;  // block tables (fp32, [6, d] each, stride in floats)
  float* mod;                        // [N, 6d]
  float* scratch;                    // 256 + 2d floats
  int d, n_blocks;
  bool bf16;
  int* set_flag = nullptr;  // non-null: the first kernel, once its dependent-launch wait has returned
                            // (every kernel before it on the stream complete), stores 1 here (release)
};
cudaError_t launch_temb(const TembArgs& a, cudaStream_t s);

// Attention.  q: [B, H, Lq, Dh]; keys/values are rows [0, Lk) of the cache
// [B, H, Lcache, Dh]; out: [B*Lq, H*Dh].  Video: keys = video tokens only;
// action: keys = [video; action] (rows [0, L_v + L_a)), split over key blocks.
struct AttnArgs {
  const void* q; const void* k; const void* v; void* out;
  int B, H, Dh, Lq, Lk, Lcache;
  int splits;        // key splits (1 = single pass)
  int ld_out = 0;    // row stride of out (0: H * Dh)
  float* ws;         // partial O / m / l when splits > 1
  int* tickets;      // B*H counters, zero on entry, left zero
};
cudaError_t launch_attention_bf16(const AttnArgs& a, cudaStream_t s);
// Sets the split kernel's shared-memory limit; call once per device before
// any launch (and never during stream capture).
cudaError_t prepare_attention_bf16();

// Joint action attention: queries q [B, H, Lq, 64] bf16 (Lq <= 64) over
// cache rows [0, Lk) of the K / V maps ([z][rows][64] bf16, box 64 x 64
// rows; (b, h) reads matrix z0 + b*H + h), out bf16 rows ld_out apart (0:
// H*64).  `splits` (1, 2, 4, 8; splits * Lq <= 279) CTAs per (b, h) form a cluster, each taking a
// contiguous key range; their partials are merged in split order in the
// cluster's shared memory.  Cache rows below `ready` must be complete before
// the launch (they are read before the dependent-launch wait); 0 makes no
// such assumption.
struct AttnJoint {
  const CUtensorMap* map_k;
  const CUtensorMap* map_v;
  int zk0, zv0;
  const void* q;
  void* out;
  int B, H, Lq, Lk, ld_out;
  int ready;
  const int* ready_flag = nullptr;  // non-null: the rows below `ready` are read before the dependent-launch
                                    // wait only if this flag reads 1 (acquire), else after it
  int splits;
  bool spread = false;  // one CTA per SM (more shared memory than it needs): for launches with the GPU to themselves
  unsigned* status;
};
cudaError_t launch_attention_joint(const AttnJoint& a, cudaStream_t s);
cudaError_t prepare_attention_joint();
// Splits for B*H (sample, head) pairs of Lq queries over Lk keys on num_sms
// SMs (the partials of all splits fit one CTA's K/V ring: splits * Lq <= 279).
int attention_joint_splits(int BH, int Lq, int Lk, int num_sms);

// Tensor-core (tcgen05) attention for video queries: one pass over keys
// [0, Lk) for 128-query tiles.  Q / K / V are 3-D TMA maps over [z][rows][64]
// bf16 (Q box 64 x 128 rows, K / V box 64 x 64 rows); (b, h) reads matrix
// z0 + b*H + h of each map.
struct AttnTc {
  const CUtensorMap* map_q;
  const CUtensorMap* map_k;
  const CUtensorMap* map_v;
  int zq0, zk0, zv0;
  int B, H, Lq, Lk;
  void* out;  // bf16 [B*Lq, H*64]
  unsigned* status;
};
cudaError_t launch_attention_tc(const AttnTc& a, cudaStream_t s);
cudaError_t prepare_attention_tc();
cudaError_t launch_attention_f32(const AttnArgs& a, cudaStream_t s);
size_t attention_ws_floats(int B, int H, int Dh, int Lq, int splits);

// Chunk input/output movers.
cudaError_t launch_init_video(const VideoIo* io, float* x, int B, int Lc, int Lvid, int d,
                              cudaStream_t s);
cudaError_t launch_init_action(const ActionIo* io, float* a_state, void* a_in, bool a_in_bf16,
                               int M, int P, int ld_in, cudaStream_t s);
cudaError_t launch_copy_out(const ActionIo* io, const float* a_state, int n, cudaStream_t s);
cudaError_t launch_set_video_io(VideoIo* dst, const VideoIo& v, cudaStream_t s);
cudaError_t launch_set_action_io(ActionIo* dst, const ActionIo& v, cudaStream_t s);

// Joint variant input construction: x_sigma = (1 - sigma) x0 + sigma eps with the
// SNR-shifted sigma computed on device from the io block.
cudaError_t launch_noise_video(const VideoIo* io, float* x_sigma, void* x_act, bool act_bf16,
                               int n_rows, int P, int ld_act, cudaStream_t s);
cudaError_t launch_noise_action(const ActionIo* io, float* a_state, void* a_in, bool a_in_bf16,
                                int M, int P, int ld_in, cudaStream_t s);

// Seeded parameters (counter-based SplitMix64 + Box-Muller, see wam.h).
// Element e of a [rows, cols] parameter is stored at out[(e / cols) * ld + e % cols].
cudaError_t launch_gen_param(uint64_t seed, uint64_t pid, size_t count, double stdv, bool ones,
                             bool round_bf16, void* out, bool out_bf16, int cols, int ld, cudaStream_t s);
cudaError_t launch_rope_table(float* cos_t, float* sin_t, int L, int Dh, cudaStream_t s);
// dst[e] = src[(e / cols) * ld + e % cols] as fp32.
cudaError_t launch_to_f32(const void* src, bool src_bf16, float* dst, size_t n, int cols, int ld, cudaStream_t s);

// ---- persistent action-expert block (action_block.cu) -------------------
// One launch = [attention of block i,] then up to five weight GEMM phases
// (out-projection, FFN up, FFN down, next block's QKV or the output map; or
// in-projection + QKV of block 0).  A phase's work units wait only on what
// they read (per-tile and per-head completion counters), never on a grid-wide
// barrier.  Batches of at most 32 action tokens, bf16.
enum : int { kBTma = 0, kBNorm = 1, kBAttn = 2 };  // B operand: TMA of an activation map / RMSNorm+modulation
                                                     // of x_a / the attention output combined from its splits
enum : int { kDepNone = 0, kDepAll = 1, kDepKRange = 2, kDepHeads = 3 };
constexpr int kActionBlockMaps = 11;
constexpr int kActionBlockPhases = 5;
constexpr int kActionBlockMaxTiles = 64;  // weight tiles of one phase (n_out <= 8192)
constexpr int kActionBlockMaxKeys = 192;  // keys per attention unit
// Tensor maps: 0 w_qkv, 1 w_o, 2 w_f1, 3 w_f2 (3-D, z = block), 4 w_in, 5 w_out,
// 6 (unused), 7 f_a, 8 a_in (box 64 x 32 rows), 9 q_a (box 64 x 128 rows),
// 10 the K/V cache (box 64 x keys-per-split rows).
struct ActionBlockMaps {
  CUtensorMap m[kActionBlockMaps];
};
// C[token m, feature n] = sum_k X[m, k] W[n, k] over W [n_out, K] (matrix z
// of map map_w), split into ks k-ranges per 128-row tile.  B = X from map
// map_b (kBTma), rms(x_a) * (ngain | 1 + nscale) + nshift with the row sums of
// squares from ss buffer ss_in (kBNorm), or the attention output (kBAttn).
// dep: what the phase's units wait for -- every tile of the previous phase
// (kDepAll), the previous phase's tiles that cover the unit's k-range
// (kDepKRange), the attention heads of the unit's k-range (kDepHeads).
// Epilogues writing x_a also write its per-tile row sums of squares into ss
// buffer ss_out (-1: none) and, when war_phase >= 0, first wait until every
// CTA has built that earlier phase's operand (it read x_a).
struct ActionGemmPhase {
  int map_w, z, n_out, K, ks;
  int bsrc, map_b, dep, ss_in, ss_out, war_phase;
  const float* nscale;
  const float* nshift;
  const float* ngain;
  int epi;  // kEpiStoreF32 / kEpiGateRes / kEpiGelu / kEpiQkv / kEpiEuler
  const float* bias;
  const float* gate;
  float* out_f32;
  __nv_bfloat16* out_act;
  int ld_out;
  const float* gq;         // QKV: per-head norm gains [A]
  const float* gk;
  __nv_bfloat16* q_out;    // [B, H, L_a, 64]
  __nv_bfloat16* k_cache;  // block base [B, H, L_tot, 64]
  __nv_bfloat16* v_cache;
  int step;                // Euler: step index into the schedule
  __nv_bfloat16* a_next;   // Euler: next in-projection input (ld a_next_ld)
  int a_next_ld;
};
struct ActionAttnPhase {
  int zk0, zv0;  // cache-map matrix index of (b = 0, h = 0) of K / V
  int splits;    // key splits of [0, Lk)
  int keys;      // keys per split (a multiple of 64, <= kActionBlockMaxKeys)
};
struct ActionBlockArgs {
  int n_gemm, has_attn;
  ActionGemmPhase g[kActionBlockPhases];
  ActionAttnPhase at;
  int Ma, La, H, A, da, Lk, cache_len, cache_off, B;
  const float* x_a;  // fp32 [Ma, da]
  float* ss;         // row sums of squares of x_a: [2][da / 128][Ma]
  const float* rope_cos;
  const float* rope_sin;
  const ActionIo* aio;
  float* ws;       // GEMM partial tiles: action_block_ws_floats (two halves, by phase parity)
  size_t ws_half;  // floats per half
  float* ws_attn;  // attention partials: action_block_attn_ws_floats
  int* cnt;        // action_block_cnt_ints: zero at first use, left zero by every launch
  int* cnt_attn;   // B * H ints, likewise
  unsigned* status;
};
// k-splits of a phase with n_out weight rows and reduction K on nsm SMs
// (fixed by the shapes, never by the grid size).
int action_block_ks(int n_out, int K, int nsm);
// Whether every CTA of a `ctas` grid holds the B k-blocks it needs.
bool action_block_fits(int n_out, int K, int ks, int ctas);
size_t action_block_ws_floats(int max_units);
size_t action_block_attn_ws_floats(int B, int H, int splits);
int action_block_cnt_ints();
// Key splits and keys per split of the attention over Lk keys for B * H heads on nsm SMs.
void action_block_attn_plan(int Lk, int bh, int nsm, int* splits, int* keys);
cudaError_t prepare_action_block();
// `ctas` <= the SM count (one CTA per SM: units wait on one another, so the whole grid must be resident).
cudaError_t launch_action_block(const ActionBlockMaps& m, const ActionBlockArgs& a, int ctas, cudaStream_t s);

// Pixel front-end: frames [B, F, C, H, W] -> patch tokens [B, F (H/p)(W/p), C p p]
// (inverse: the other way).
cudaError_t launch_patchify(const float* src, float* dst, int B, int F, int C, int H, int W, int p, bool inverse,
                            cudaStream_t s);

// TACD target forward: a_t = (1 - t) a_clean + t eps; and the targets
// u_TA, v_student, u_CD (any may be null) plus losses[3] = L_TA, L_CD,
// L_CD + lambda L_TA from the teacher end state, the student and EMA endpoints.
cudaError_t launch_tacd_noise(const float* a_clean, const float* eps, float t, float* a_t, int n, cudaStream_t s);
cudaError_t launch_tacd_targets(const float* a_t, const float* a0_teacher, const float* f_student,
                                const float* f_ema, float t, float lambda, int B, int per_sample, float* u_ta,
                                float* v_student, float* u_cd, float* losses, cudaStream_t s);

// TMA tensor-map creation (driver entry point resolved at run time).
bool make_tmap_3d(CUtensorMap* map, const void* base, int K, int rows, int nmat, size_t mat_stride_bytes,
                  int box_rows);
// General 3-D map with the 128-byte swizzle: elem_bytes 2 (bf16) or 4 (fp32),
// dims (inner, rows, nmat), box (box_inner, box_rows, 1).
bool make_tmap_sw128(CUtensorMap* map, const void* base, int elem_bytes, int inner, int rows, int nmat,
                     size_t mat_stride_bytes, int box_inner, int box_rows);

}  // namespace wam
