// C ABI of the MoT world-action-model forward: context, seeded parameters,
// the sequential and Cross-Expert Wavefront Pipeline (CEWP) schedules, CUDA
// graph capture, and the single-operation entry points.
//
// Schedules (RealtimeWAM summary page, sections 核心方法 / 方法步骤详情;
// tokendh.com article, CEWP section).  A DiT block splits into P_i (norm +
// merged QKV projection with QK-norm, RoPE and the K/V publish fused into its
// epilogue), Attn_i and R_i (out-projection + FFN).  CEWP puts the video
// expert on one stream and the action expert on another: the video stream
// records event e_i right after P^v_i, the action stream waits on e_i right
// before Attn^a_i and on nothing else.  The sequential schedule enqueues the
// same kernels, with the same launch configurations, on one stream -- the two
// differ only in order, so their results are bitwise identical (every kernel
// is deterministic; split reductions use a fixed order).
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <initializer_list>
#include <map>
#include <memory>
#include <string>
#include <vector>

#include "../../include/wam.h"
#include "kernels.h"

using namespace wam;

namespace {

struct PEntry {
  std::string name;
  int rows, cols, ld;
  bool matrix, ones;
  size_t off;  // elements into wmat (matrix) or wvec (vector)
  // LoRA B factors live inside their layer's weight matrix: columns
  // [col_off, col_off + cols) of matrix `alias` (same ld), see add_expert
  int alias = -1, col_off = 0;
  size_t count() const { return (size_t)rows * cols; }
};

// Per-block entry order (must match the generation order below).
enum BlkLocal {
  kT = 0, kQkvW, kQkvB, kQnG, kKnG, kOW, kOB, kF1W, kF1B, kF2W, kF2B,
  kQkvLa, kQkvLb, kOLa, kOLb, kF1La, kF1Lb, kF2La, kF2Lb
};

struct ExpertIdx {
  int t1w, t1b, t2w, t2b, modw, modb;
  int inw = -1, inb = -1, fng = -1, outw = -1, outb = -1;
  int blk0 = -1, per_blk = 0;
};

struct Dims {
  int N, dv, da, H, Dh, A, Fv, Fa, Lc, Lvid, Lv, La, Pa, Pv, B, r, Ltot, Mv, Ma, Kin;
  // row strides of the action GEMM inputs h_a, o_a, f_a: each row carries the
  // layer input and, with LoRA, the r columns of s x A^T after it
  int lh, lo, lf;
  bool bf16;
};

struct GemmPlan {
  int bn = 128, splits = 1, max_ctas = 0;
  bool pair = false;    // normal orientation, bn 256: CTA pairs (2-SM MMA)
  bool csplit = false;  // normal orientation: clusters of two, split tiles finished in column halves
  int cred = 0;         // swapped: clusters of `splits` CTAs sum each tile's pieces in shared memory
};

}  // namespace

struct wam_ctx {
  wam_config cfg{};
  Dims d{};
  int device = 0;
  std::vector<PEntry> params;
  ExpertIdx ev{}, ea{};
  void* wmat = nullptr;
  float* wvec = nullptr;
  size_t wmat_elems = 0, wvec_elems = 0;
  size_t esz = 2;  // bytes per activation / matrix element

  // activations
  float *x_v = nullptr, *x_a = nullptr, *a_state = nullptr, *x_sigma = nullptr;
  void *h_v = nullptr, *q_v = nullptr, *o_v = nullptr, *f_v = nullptr, *x_vin = nullptr;
  void *h_a = nullptr, *q_a = nullptr, *o_a = nullptr, *f_a = nullptr, *a_in = nullptr;
  float *qkv_tmp_v = nullptr, *qkv_tmp_a = nullptr;  // fp32 path only
  void* kv = nullptr;                                 // [N][2][B][H][Ltot][Dh]
  float *mod_v = nullptr, *mod_a = nullptr, *temb_v = nullptr, *temb_a = nullptr;
  float *rope_cos = nullptr, *rope_sin = nullptr;
  float* zero_r = nullptr;   // r zeros: the (absent) bias of the LoRA down-projection
  float* ws_gemm = nullptr;  // action-stream GEMM partial tiles / tickets
  int* tk_gemm = nullptr;
  float* ws_gemm_v = nullptr;  // video-stream GEMM partial tiles / tickets (the streams overlap)
  int* tk_gemm_v = nullptr;
  size_t tk_gemm_bytes = 0, tk_gemm_v_bytes = 0;
  int* na_cnt = nullptr;     // video norm prologue row counters (taken, done, CTAs out)
  bool fuse_norm_v = false;  // the video QKV / FFN-up GEMMs normalise their own A rows
  float* ws_attn = nullptr;
  int* tk_attn = nullptr;
  unsigned* status = nullptr;
  VideoIo *vio_chunk = nullptr, *vio_eager = nullptr;
  ActionIo *aio_chunk = nullptr, *aio_eager = nullptr;
  VideoIo vio_shadow{};
  ActionIo aio_shadow{};
  bool vio_valid = false, aio_valid = false;
  float *h_video = nullptr, *h_cond = nullptr, *h_noise = nullptr, *h_out = nullptr;  // host-API staging
  float *j_vout = nullptr, *j_aout = nullptr;
  // TACD target forward (allocated on first use): a_t, teacher state at s,
  // teacher end state, student and EMA endpoints; the schedule block of its runs
  float *td_at = nullptr, *td_as = nullptr, *td_a0 = nullptr, *td_fs = nullptr, *td_fe = nullptr;
  ActionIo* aio_tacd = nullptr;

  // plans
  GemmPlan p_v_qkv, p_v_o, p_v_f1, p_v_f2, p_v_in, p_v_out;
  GemmPlan p_a_in, p_a_qkv, p_a_o, p_a_f1, p_a_f2, p_a_out;
  // Euler steps j >= 1 (no video kernels beside them): splits over clusters
  GemmPlan p_a_qkv_l, p_a_o_l, p_a_f1_l, p_a_f2_l;
  GemmPlan p_u_qkv, p_u_o, p_u_f1, p_u_f2;  // LoRA down-projections u = s x A^T
  int attn_splits = 1;
  int attn_joint_splits = 0;  // joint action attention on clusters (0: the split-KV kernel)
  bool attn_spread = true;    // ... one CTA per SM (no video kernels beside it)
  bool attn_prefetch = false; // ... its video rows may be read before its dependent-launch wait (kv_flag)
  int* kv_flag = nullptr;     // 1 once a step j >= 1 has begun: every video block's K/V is complete
  bool kv_flag_clean = true;  // host: no sequence that may set kv_flag was left without its clearing
  // The action expert's norms run inside the GEMM that consumes them (opt-in;
  // the tokens must fit one 32/64-wide tile and K <= 1024).
  bool fuse_norm_a = false;
  // Persistent action-block path (action_block.cu): one launch per action
  // block; grid sizes for launches that may overlap the video expert (CEWP
  // first step, eager action steps) and for the rest.
  bool ab_on = false;
  int ab_ctas = 0, ab_ctas_overlap = 0;
  int ab_ks_in = 1, ab_ks_qkv = 1, ab_ks_o = 1, ab_ks_f1 = 1, ab_ks_f2 = 1, ab_ks_out = 1, ab_splits = 1, ab_keys = 64;
  ActionBlockMaps ab_maps;
  float *ab_ws = nullptr, *ab_ws_attn = nullptr, *ab_ss = nullptr;
  size_t ab_ws_half = 0;
  int *ab_cnt = nullptr, *ab_cnt_attn = nullptr;

  // TMA maps
  CUtensorMap m_hv, m_ov, m_fv, m_xvin, m_w_qkv_v, m_w_o_v, m_w_f1_v, m_w_f2_v, m_w_vin, m_w_vout;
  CUtensorMap m_w_in, m_w_qkv_a, m_w_o_a, m_w_f1_a, m_w_f2_a, m_w_out, m_ain, m_ha, m_oa, m_fa;
  CUtensorMap m_la_qkv, m_la_o, m_la_f1, m_la_f2;  // LoRA A factors [r, in] per block
  CUtensorMap m_qv, m_cache;  // video-attention operands
  CUtensorMap m_qa128, m_cache_ab;  // action-block attention operands (Q: 128-row box; K/V: keys per split)
  // video GEMM outputs (TMA stores, 32-row boxes): x_v fp32, f_v bf16, Q, the K/V cache
  CUtensorMap m_xv_out, m_fv_out, m_qv_out, m_cache_out;

  // events and streams
  std::vector<cudaEvent_t> ev_kv, ev_kv_cap, ev_used;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr, ev_pre = nullptr, ev_post = nullptr;
  cudaStream_t cap_v = nullptr, cap_a = nullptr;
  std::map<long long, cudaGraphExec_t> graphs;
  std::map<long long, int> launch_counts;
  bool video_done = false;
  int launches = 0;
  std::string last_error;
  // device-memory budget of the context (WAM_DEVICE_MEMORY_LIMIT, bytes; 0 = none)
  size_t mem_limit = 0, mem_used = 0;

  // per-launch timing (wam_profile_chunk)
  bool prof_on = false;
  int cur_cls = 0;
  struct ProfRec {
    int cls;
    cudaEvent_t a, b;
  };
  std::vector<ProfRec> prof;
  std::vector<cudaEvent_t> prof_pool;
  size_t prof_next = 0;

  // wavefront trace (wam_trace_chunk): timing events at block boundaries
  bool trace_on = false;
  struct TraceRec {
    int kind, block, step;
    cudaEvent_t e;
  };
  std::vector<TraceRec> trace;
  std::vector<cudaEvent_t> trace_pool;
  int trace_step = 0;
};

namespace {

wam_status fail(wam_ctx* c, wam_status s, const char* fmt, ...) {
  if (c) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    c->last_error = buf;
  }
  return s;
}

#define CK(expr)                                                                              \
  do {                                                                                        \
    cudaError_t e_ = (expr);                                                                  \
    if (e_ != cudaSuccess) return fail(c, WAM_ERR_CUDA, "%s: %s (%s:%d)", #expr,              \
                                       cudaGetErrorString(e_), __FILE__, __LINE__);           \
  } while (0)

// Records a timing event pair around the launches inside its scope when the
// context is profiling (eager, one stream), tagged with the current class.
struct ProfScope {
  wam_ctx* c;
  cudaStream_t s;
  cudaEvent_t b = nullptr;
  ProfScope(wam_ctx* c_, cudaStream_t s_) : c(c_), s(s_) {
    if (!c->prof_on) return;
    while (c->prof_pool.size() < c->prof_next + 2) {
      cudaEvent_t e;
      if (cudaEventCreate(&e) != cudaSuccess) return;
      c->prof_pool.push_back(e);
    }
    cudaEvent_t a = c->prof_pool[c->prof_next++];
    b = c->prof_pool[c->prof_next++];
    cudaEventRecordWithFlags(a, s, cudaEventRecordExternal);
    c->prof.push_back({c->cur_cls, a, b});
  }
  ~ProfScope() {
    if (b) cudaEventRecordWithFlags(b, s, cudaEventRecordExternal);
  }
};

// Records a timing event of `kind` for block i on stream s when the context is
// tracing (wam_trace_chunk); a no-op otherwise.
void trace_mark(wam_ctx* c, cudaStream_t s, int kind, int i) {
  if (!c->trace_on) return;
  if (c->trace.size() >= c->trace_pool.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return;
    c->trace_pool.push_back(e);
  }
  cudaEvent_t e = c->trace_pool[c->trace.size()];
  cudaEventRecordWithFlags(e, s, cudaEventRecordExternal);
  c->trace.push_back({kind, i, c->trace_step, e});
}

// ------------------------------------------------------------ parameters --
void add_expert(wam_ctx* c, bool video) {
  const Dims& d = c->d;
  const int dm = video ? d.dv : d.da, F = video ? d.Fv : d.Fa, A = d.A;
  const std::string p = video ? "video." : "action.";
  ExpertIdx& ix = video ? c->ev : c->ea;
  auto add = [&](const std::string& n, int rows, int cols, bool matrix, bool ones) {
    PEntry e;
    e.name = n;
    e.rows = rows;
    e.cols = cols;
    e.matrix = matrix;
    e.ones = ones;
    e.ld = (matrix && d.bf16) ? (cols + 63) / 64 * 64 : cols;
    e.off = 0;
    c->params.push_back(e);
    return (int)c->params.size() - 1;
  };
  ix.t1w = add(p + "t1.w", dm, 256, true, false);
  ix.t1b = add(p + "t1.b", 1, dm, false, false);
  ix.t2w = add(p + "t2.w", dm, dm, true, false);
  ix.t2b = add(p + "t2.b", 1, dm, false, false);
  ix.modw = add(p + "mod.w", 6 * dm, dm, true, false);
  ix.modb = add(p + "mod.b", 1, 6 * dm, false, false);
  if (video && d.Pv > 0) {
    ix.inw = add(p + "in.w", dm, d.Pv, true, false);
    ix.inb = add(p + "in.b", 1, dm, false, false);
  }
  if (!video) {
    ix.inw = add(p + "in.w", dm, d.Pa, true, false);
    ix.inb = add(p + "in.b", 1, dm, false, false);
  }
  const bool lora = !video && d.r > 0;
  for (int i = 0; i < d.N; ++i) {
    const std::string b = p + "blk" + std::to_string(i) + ".";
    const int first = add(b + "T", 6, dm, false, false);
    if (i == 0) ix.blk0 = first;
    const int wq = add(b + "qkv.w", 3 * A, dm, true, false);
    add(b + "qkv.b", 1, 3 * A, false, false);
    add(b + "qn.g", 1, A, false, true);
    add(b + "kn.g", 1, A, false, true);
    const int wo = add(b + "o.w", dm, A, true, false);
    add(b + "o.b", 1, dm, false, false);
    const int w1 = add(b + "ffn1.w", F, dm, true, false);
    add(b + "ffn1.b", 1, F, false, false);
    const int w2 = add(b + "ffn2.w", dm, F, true, false);
    add(b + "ffn2.b", 1, dm, false, false);
    if (lora) {
      // Unmerged LoRA y = x W^T + b + s (x A^T) B^T as one GEMM over the
      // concatenated reduction [x | s x A^T] . [W | B]^T: B sits in columns
      // [K, K + r) of W's rows (W's leading dimension grows by r).
      auto lb = [&](const std::string& n, int w) {
        const int k = c->params[w].ld, rows = c->params[w].rows;
        c->params[w].ld = k + d.r;
        const int e = add(n, rows, d.r, true, false);  // (may reallocate the table)
        c->params[e].ld = k + d.r;
        c->params[e].alias = w;
        c->params[e].col_off = k;
      };
      add(b + "qkv.la", d.r, dm, true, false);
      lb(b + "qkv.lb", wq);
      add(b + "o.la", d.r, A, true, false);
      lb(b + "o.lb", wo);
      add(b + "ffn1.la", d.r, dm, true, false);
      lb(b + "ffn1.lb", w1);
      add(b + "ffn2.la", d.r, F, true, false);
      lb(b + "ffn2.lb", w2);
    }
    if (i == 0) ix.per_blk = (int)c->params.size() - first;
  }
  if (video && c->cfg.video_has_output) {
    ix.fng = add(p + "fn.g", 1, dm, false, true);
    ix.outw = add(p + "out.w", d.Pv, dm, true, false);
    ix.outb = add(p + "out.b", 1, d.Pv, false, false);
  }
  if (!video) {
    ix.fng = add(p + "fn.g", 1, dm, false, true);
    ix.outw = add(p + "out.w", d.Pa, dm, true, false);
    ix.outb = add(p + "out.b", 1, d.Pa, false, false);
  }
}

void layout_params(wam_ctx* c) {
  size_t om = 0, ov = 0;
  for (auto& e : c->params) {
    if (e.matrix && e.alias >= 0) {
      e.off = c->params[e.alias].off + e.col_off;
    } else if (e.matrix) {
      e.off = om;
      om += ((size_t)e.rows * e.ld + 127) / 128 * 128;
    } else {
      e.off = ov;
      ov += (e.count() + 63) / 64 * 64;
    }
  }
  c->wmat_elems = om;
  c->wvec_elems = ov;
}

inline int blk(const ExpertIdx& x, int i, int local) { return x.blk0 + i * x.per_blk + local; }
inline void* matp(wam_ctx* c, int idx) { return (char*)c->wmat + c->params[idx].off * c->esz; }
inline float* vecp(wam_ctx* c, int idx) { return c->wvec + c->params[idx].off; }
inline size_t blk_stride_bytes(wam_ctx* c, const ExpertIdx& x, int local) {
  if (c->d.N < 2) return 0;
  return (c->params[blk(x, 1, local)].off - c->params[blk(x, 0, local)].off) * c->esz;
}
inline void* kcache(wam_ctx* c, int i) {
  const size_t per = (size_t)c->d.B * c->d.H * c->d.Ltot * c->d.Dh;
  return (char*)c->kv + (size_t)(2 * i) * per * c->esz;
}
inline void* vcache(wam_ctx* c, int i) {
  const size_t per = (size_t)c->d.B * c->d.H * c->d.Ltot * c->d.Dh;
  return (char*)c->kv + (size_t)(2 * i + 1) * per * c->esz;
}

#define RET(expr)                       \
  do {                                  \
    wam_status r_ = (expr);             \
    if (r_ != WAM_OK) return r_;        \
  } while (0)

// ------------------------------------------------------------- planning ---
GemmPlan plan_swap(int rows_w, int tokens, int K, int bn, bool fused_norm, int target_ctas, bool cred = false,
                   int wide_splits = 0) {
  GemmPlan p;
  p.bn = bn;
  const int tiles = ((rows_w + 127) / 128) * ((tokens + bn - 1) / bn);
  const int kb = (K + 63) / 64;
  int s = (target_ctas + tiles - 1) / tiles;
  const int min_kb = 3;  // keep each split a few k-blocks deep
  if (s > kb / min_kb) s = kb / min_kb;
  // With 24 or more feature tiles the weights already stream from as many
  // SMs; splits summed through global partials only added the hand-off
  // (action QKV / FFN-up at 32 tokens: 4 splits 16.6 us, none 14.5 us per
  // launch in the 10-step chunk), so such a GEMM splits only over clusters
  // (wide_splits CTAs summing in shared memory), else not at all.
  if (tiles >= 24) s = cred && wide_splits > 1 ? wide_splits : 1;
  // a tile takes at most splits + 1 pieces; the last one's partner partials
  // must fit its operand ring for the fast reduction
  const int cap = tc_gemm_ring_partials(bn, true, fused_norm);
  if (s > cap) s = cap;
  if (s < 1) s = 1;
  p.splits = s;
  // Cluster reduction: a split count that divides the k-blocks and bn / 4
  // (whole 4-column slices per CTA), at most 8 (a portable cluster), no less than
  // half the stream-K choice (the weight stream keeps most of its SMs).  The
  // pieces are then summed in shared memory instead of through global
  // partials and tickets (action out-proj / FFN-down at 32 tokens: 8 splits).
  if (cred && !fused_norm && s > 1) {
    int S = 0;
    for (int c = std::min({8, bn / 4, std::max(s, 2)}); c >= 2; --c)
      if (kb % c == 0 && (bn / 4) % c == 0) {
        S = c;
        break;
      }
    if (S >= 2 && 2 * S >= std::min(s, 8)) {
      p.splits = S;
      p.cred = S;
    }
  }
  if (tiles >= 24 && p.cred == 0) p.splits = 1;
  return p;
}

// --------------------------------------------------------- GEMM wrappers --
wam_status run_tc(wam_ctx* c, const CUtensorMap& A, const CUtensorMap& Bm, int rows_a, int rows_b, int K, int z_a,
                  int z_b, const GemmPlan& p, bool swap, const EpiArgs& e, cudaStream_t s, bool video) {
  TcGemm g;
  g.map_a = &A;
  g.map_b = &Bm;
  g.rows_a = rows_a;
  g.rows_b = rows_b;
  g.K = K;
  g.z_a = z_a;
  g.z_b = z_b;
  g.bn = p.bn;
  g.splits = p.splits;
  g.swap = swap;
  g.max_ctas = p.max_ctas;
  g.pair = p.pair;
  g.csplit = p.csplit;
  g.cred = p.cred;
  g.ws = video ? c->ws_gemm_v : c->ws_gemm;
  g.tickets = video ? c->tk_gemm_v : c->tk_gemm;
  g.status = c->status;
  c->launches++;
  CK(launch_tc_gemm(g, e, s));
  return WAM_OK;
}

EpiArgs epi_base(int kind, const float* bias, float* out_f32, void* out_act, int ld) {
  EpiArgs e;
  e.kind = kind;
  e.bias = bias;
  e.out_f32 = out_f32;
  e.out_act = out_act;
  e.ld_out = ld;
  return e;
}

EpiArgs epi_qkv(wam_ctx* c, bool video, int i) {
  const Dims& d = c->d;
  const ExpertIdx& x = video ? c->ev : c->ea;
  EpiArgs e = epi_base(kEpiQkv, vecp(c, blk(x, i, kQkvB)), nullptr, nullptr, 0);
  e.gq = vecp(c, blk(x, i, kQnG));
  e.gk = vecp(c, blk(x, i, kKnG));
  e.rope_cos = c->rope_cos;
  e.rope_sin = c->rope_sin;
  e.q_out = video ? c->q_v : c->q_a;
  e.k_cache = kcache(c, i);
  e.v_cache = vcache(c, i);
  e.seq_len = video ? d.Lv : d.La;
  e.cache_len = d.Ltot;
  e.cache_off = video ? 0 : d.Lv;
  e.n_heads = d.H;
  e.head_dim = d.Dh;
  e.attn_dim = d.A;
  return e;
}

// Linear layer of expert `video` block i (or a non-block layer when i < 0),
// dispatched to the tcgen05 path (bf16) or the SIMT path (fp32).
struct Lin {
  const CUtensorMap* map_w;  // weight map (bf16)
  const CUtensorMap* map_x;  // activation map (bf16)
  const void* w;             // fp32 path: weight pointer
  const void* x;             // activation pointer (rows ldx apart; 0: K)
  int n_out, K;              // output features, reduction length
  int z;                     // block index in the weight map
  const GemmPlan* plan;
  int ldx = 0;
  // unmerged LoRA (action expert): the A factor [r, K] of this layer
  const CUtensorMap* map_la = nullptr;
  const void* la = nullptr;
  const GemmPlan* plan_u = nullptr;
};

wam_status linear(wam_ctx* c, bool video, const Lin& L, int M, const EpiArgs& e_in, float* qkv_tmp, cudaStream_t s) {
  const Dims& d = c->d;
  ProfScope ps(c, s);
  const int ldx = L.ldx ? L.ldx : L.K;
  int K = L.K;
  if (L.la) {
    // LoRA: u = s x A^T into columns [K, K + r) of the input rows, then one
    // GEMM over the concatenated reduction [x | u] . [W | B]^T
    EpiArgs eu = epi_base(kEpiScaleAct, c->zero_r, nullptr, (char*)L.x + (size_t)L.K * c->esz, ldx);
    eu.scale = c->cfg.lora_scale;
    if (d.bf16) {
      RET(run_tc(c, *L.map_la, *L.map_x, d.r, M, L.K, L.z, 0, *L.plan_u, true, eu, s, false));
    } else {
      c->launches++;
      CK(launch_f32_gemm((const float*)L.x, ldx, (const float*)L.la, M, d.r, L.K, eu, s));
    }
    K += d.r;
  }
  if (d.bf16) {
    if (video) {  // tokens on TMEM lanes; outputs leave through TMA stores
      EpiArgs e = e_in;
      if (e.kind == kEpiQkv) {
        e.map_o = &c->m_qv_out;
        e.map_o2 = &c->m_cache_out;
        e.zq0 = 0;
        e.zk0 = 2 * L.z * d.B * d.H;
        e.zv0 = (2 * L.z + 1) * d.B * d.H;
      } else if (e.kind == kEpiGelu) {
        e.map_o = &c->m_fv_out;
      } else if (e.kind == kEpiStoreF32 || e.kind == kEpiGateRes) {
        e.map_o = &c->m_xv_out;
      }
      return run_tc(c, *L.map_x, *L.map_w, M, L.n_out, K, 0, L.z, *L.plan, false, e, s, true);
    }
    return run_tc(c, *L.map_w, *L.map_x, L.n_out, M, K, L.z, 0, *L.plan, true, e_in, s, false);
  }
  if (e_in.kind == kEpiQkv) {
    EpiArgs st = epi_base(kEpiStoreF32, e_in.bias, qkv_tmp, nullptr, 3 * d.A);
    c->launches++;
    CK(launch_f32_gemm((const float*)L.x, ldx, (const float*)L.w, M, L.n_out, K, st, s));
    c->launches++;
    CK(launch_qkv_post_f32(qkv_tmp, M, e_in, s));
    return WAM_OK;
  }
  c->launches++;
  CK(launch_f32_gemm((const float*)L.x, ldx, (const float*)L.w, M, L.n_out, K, e_in, s));
  return WAM_OK;
}

wam_status norm(wam_ctx* c, const float* x, void* h, int M, int dm, const float* sc, const float* sh, const float* g,
                cudaStream_t s, int ldh = 0) {
  c->launches++;
  ProfScope ps(c, s);
  CK(launch_norm_mod(x, h, c->d.bf16, M, dm, sc, sh, g, s, ldh));
  return WAM_OK;
}

// Action-expert linear layer whose input is h = rms(x_a) (gain or 1 + scale)
// + shift: the norm is computed inside the GEMM when it fits, otherwise by
// the norm kernel into h_a first.  `cls` is the profile class of the GEMM.
wam_status norm_linear(wam_ctx* c, const Lin& L, EpiArgs e, const float* sc, const float* sh, const float* gain,
                       int cls, cudaStream_t s);

wam_status temb(wam_ctx* c, bool video, const float* t, cudaStream_t s, int* set_flag = nullptr) {
  const ExpertIdx& x = video ? c->ev : c->ea;
  TembArgs a;
  a.t = t;
  a.w1 = matp(c, x.t1w);
  a.b1 = vecp(c, x.t1b);
  a.w2 = matp(c, x.t2w);
  a.b2 = vecp(c, x.t2b);
  a.wm = matp(c, x.modw);
  a.bm = vecp(c, x.modb);
  a.T0 = vecp(c, blk(x, 0, kT));
  a.T_stride = c->d.N > 1 ? c->params[blk(x, 1, kT)].off - c->params[blk(x, 0, kT)].off : 0;
  a.mod = video ? c->mod_v : c->mod_a;
  a.scratch = video ? c->temb_v : c->temb_a;
  a.d = video ? c->d.dv : c->d.da;
  a.n_blocks = c->d.N;
  a.bf16 = c->d.bf16;
  a.set_flag = set_flag;
  c->launches += 3;
  ProfScope ps(c, s);
  CK(launch_temb(a, s));
  return WAM_OK;
}

wam_status attention(wam_ctx* c, bool video, int i, cudaStream_t s) {
  const Dims& d = c->d;
  AttnArgs a;
  a.q = video ? c->q_v : c->q_a;
  a.k = kcache(c, i);
  a.v = vcache(c, i);
  a.out = video ? c->o_v : c->o_a;
  a.B = d.B;
  a.H = d.H;
  a.Dh = d.Dh;
  a.Lq = video ? d.Lv : d.La;
  a.Lk = video ? d.Lv : d.Lv + d.La;
  a.Lcache = d.Ltot;
  a.splits = video ? 1 : c->attn_splits;
  a.ld_out = video ? 0 : d.lo;
  a.ws = c->ws_attn;
  a.tickets = c->tk_attn;
  c->launches++;
  ProfScope ps(c, s);
  if (d.bf16 && video) {
    AttnTc t;
    t.map_q = &c->m_qv;
    t.map_k = &c->m_cache;
    t.map_v = &c->m_cache;
    t.zq0 = 0;
    t.zk0 = (2 * i) * d.B * d.H;
    t.zv0 = (2 * i + 1) * d.B * d.H;
    t.B = d.B;
    t.H = d.H;
    t.Lq = d.Lv;
    t.Lk = d.Lv;
    t.out = c->o_v;
    t.status = c->status;
    CK(launch_attention_tc(t, s));
    return WAM_OK;
  }
  if (d.bf16 && c->attn_joint_splits > 0) {
    // action queries over [K^v_i; K^a_i].  Nothing is read before the
    // dependent-launch wait: under stream capture the edge from the video
    // stream's event also arrives as a programmatic dependency, so the video
    // rows too are complete only after the wait (read earlier, the captured
    // CEWP chunk differed from the sequential one).
    AttnJoint t;
    t.map_k = &c->m_cache;
    t.map_v = &c->m_cache;
    t.zk0 = (2 * i) * d.B * d.H;
    t.zv0 = (2 * i + 1) * d.B * d.H;
    t.q = c->q_a;
    t.out = c->o_a;
    t.B = d.B;
    t.H = d.H;
    t.Lq = d.La;
    t.Lk = d.Lv + d.La;
    t.ld_out = d.lo;
    t.ready = c->attn_prefetch ? d.Lv : 0;
    t.ready_flag = c->attn_prefetch ? c->kv_flag : nullptr;
    t.splits = c->attn_joint_splits;
    t.spread = c->attn_spread;
    t.status = c->status;
    CK(launch_attention_joint(t, s));
    return WAM_OK;
  }
  CK(d.bf16 ? launch_attention_bf16(a, s) : launch_attention_f32(a, s));
  return WAM_OK;
}

wam_status norm_linear(wam_ctx* c, const Lin& L, EpiArgs e, const float* sc, const float* sh, const float* gain,
                       int cls, cudaStream_t s) {
  const Dims& d = c->d;
  if (c->fuse_norm_a) {
    e.nb_x = c->x_a;
    e.nb_scale = sc;
    e.nb_shift = sh;
    e.nb_gain = gain;
  } else {
    c->cur_cls = WAM_PROF_ACTION_NORM;
    RET(norm(c, c->x_a, c->h_a, d.Ma, d.da, sc, sh, gain, s, d.lh));
  }
  c->cur_cls = cls;
  return linear(c, false, L, d.Ma, e, c->qkv_tmp_a, s);
}

// ------------------------------------------------------------- experts ----
// Video expert: P^v_i -> record(e_i) -> Attn^v_i -> R^v_i for every block.
// The video expert's N DiT blocks on x_v at the modulation in mod_v:
// P^v_i -> record(e_i) -> Attn^v_i -> R^v_i.
wam_status enqueue_video_blocks(wam_ctx* c, cudaStream_t s, cudaEvent_t* ev_ready, bool war_waits) {
  const Dims& d = c->d;
  const ExpertIdx& x = c->ev;
  const bool has_out = c->cfg.video_has_output != 0;
  for (int i = 0; i < d.N; ++i) {
    const float* mod = c->mod_v + (size_t)i * 6 * d.dv;
    if (war_waits) CK(cudaStreamWaitEvent(s, c->ev_used[i], 0));
    // the A operand h_v = norm(x_v) with the block's modulation: in the GEMM's
    // own prologue (fused), or by the norm kernel
    auto norm_a = [&](EpiArgs& e, const float* scale, const float* shift) -> wam_status {
      if (c->fuse_norm_v) {
        e.na_x = c->x_v;
        e.na_scale = scale;
        e.na_shift = shift;
        e.na_h = c->h_v;
        e.na_cnt = c->na_cnt;
        return WAM_OK;
      }
      c->cur_cls = WAM_PROF_VIDEO_NORM;
      return norm(c, c->x_v, c->h_v, d.Mv, d.dv, scale, shift, nullptr, s);
    };
    EpiArgs eq = epi_qkv(c, true, i);
    RET(norm_a(eq, mod + d.dv, mod));
    c->cur_cls = WAM_PROF_VIDEO_QKV;
    Lin Lq{&c->m_w_qkv_v, &c->m_hv, matp(c, blk(x, i, kQkvW)), c->h_v, 3 * d.A, d.dv, i, &c->p_v_qkv};
    RET(linear(c, true, Lq, d.Mv, eq, c->qkv_tmp_v, s));
    // (the trace mark first: an action-side mark after the wait on e_i then
    // depends on it, so the recorded order is the schedule's)
    trace_mark(c, s, WAM_TRACE_VIDEO_KV, i);
    if (ev_ready) CK(cudaEventRecord(ev_ready[i], s));
    if (i == d.N - 1 && !has_out) break;
    c->cur_cls = WAM_PROF_VIDEO_ATTN;
    RET(attention(c, true, i, s));
    c->cur_cls = WAM_PROF_VIDEO_OPROJ;
    EpiArgs eo = epi_base(kEpiGateRes, vecp(c, blk(x, i, kOB)), c->x_v, nullptr, d.dv);
    eo.gate = mod + 2 * d.dv;
    Lin Lo{&c->m_w_o_v, &c->m_ov, matp(c, blk(x, i, kOW)), c->o_v, d.dv, d.A, i, &c->p_v_o};
    RET(linear(c, true, Lo, d.Mv, eo, nullptr, s));
    EpiArgs e1 = epi_base(kEpiGelu, vecp(c, blk(x, i, kF1B)), nullptr, c->f_v, d.Fv);
    RET(norm_a(e1, mod + 4 * d.dv, mod + 3 * d.dv));
    c->cur_cls = WAM_PROF_VIDEO_FFN_UP;
    Lin L1{&c->m_w_f1_v, &c->m_hv, matp(c, blk(x, i, kF1W)), c->h_v, d.Fv, d.dv, i, &c->p_v_f1};
    RET(linear(c, true, L1, d.Mv, e1, nullptr, s));
    c->cur_cls = WAM_PROF_VIDEO_FFN_DOWN;
    EpiArgs e2 = epi_base(kEpiGateRes, vecp(c, blk(x, i, kF2B)), c->x_v, nullptr, d.dv);
    e2.gate = mod + 5 * d.dv;
    Lin L2{&c->m_w_f2_v, &c->m_fv, matp(c, blk(x, i, kF2W)), c->f_v, d.dv, d.Fv, i, &c->p_v_f2};
    RET(linear(c, true, L2, d.Mv, e2, nullptr, s));
    trace_mark(c, s, WAM_TRACE_VIDEO_END, i);
  }
  return WAM_OK;
}

// Video expert: P^v_i -> record(e_i) -> Attn^v_i -> R^v_i for every block.
// n_video > 0: the multi-step video expert -- the patch latents start at
// io->video scaled by the level io->t (1: pure noise), then n_video passes,
// each one forward at level io->vsched[j] followed by the Euler step of the
// latents; only the last pass publishes e_i (the action expert reads its
// K/V), only the first waits for the previous chunk's consumption events.
wam_status enqueue_video(wam_ctx* c, cudaStream_t s, const VideoIo* io, bool joint, cudaEvent_t* ev_ready,
                         bool war_waits, int n_video = 0) {
  const Dims& d = c->d;
  const ExpertIdx& x = c->ev;
  c->cur_cls = WAM_PROF_VIDEO_IO;
  if (joint || n_video > 0) {
    c->launches++;
    ProfScope ps(c, s);
    CK(launch_noise_video(io, c->x_sigma, d.bf16 ? c->x_vin : c->x_sigma, d.bf16, d.Mv, d.Pv, d.Pv, s));
  } else {
    c->launches++;
    ProfScope ps(c, s);
    CK(launch_init_video(io, c->x_v, d.B, d.Lc, d.Lvid, d.dv, s));
  }
  const int passes = n_video > 0 ? n_video : 1;
  for (int j = 0; j < passes; ++j) {
    if (joint || n_video > 0) {
      c->cur_cls = WAM_PROF_VIDEO_IO;
      Lin L{&c->m_w_vin, &c->m_xvin, matp(c, x.inw), c->x_sigma, d.dv, d.Pv, 0, &c->p_v_in};
      RET(linear(c, true, L, d.Mv, epi_base(kEpiStoreF32, vecp(c, x.inb), c->x_v, nullptr, d.dv), nullptr, s));
    }
    c->cur_cls = WAM_PROF_VIDEO_TEMB;
    RET(temb(c, true, n_video > 0 ? &io->vsched[j] : &io->t, s));
    RET(enqueue_video_blocks(c, s, j == passes - 1 ? ev_ready : nullptr, war_waits && j == 0));
    if (joint || n_video > 0) {
      c->cur_cls = WAM_PROF_VIDEO_IO;
      RET(norm(c, c->x_v, c->h_v, d.Mv, d.dv, nullptr, nullptr, vecp(c, x.fng), s));
      EpiArgs eo;
      if (n_video > 0) {
        eo = epi_base(kEpiVideoEuler, vecp(c, x.outb), c->x_sigma, d.bf16 ? c->x_vin : nullptr, d.Pv);
        eo.step = j;
        eo.a_next_ld = d.Pv;
      } else {
        eo = epi_base(kEpiVideoOut, vecp(c, x.outb), nullptr, nullptr, d.Pv);
        eo.x_sigma = c->x_sigma;
      }
      eo.vio = io;
      Lin Lout{&c->m_w_vout, &c->m_hv, matp(c, x.outw), c->h_v, d.Pv, d.dv, 0, &c->p_v_out};
      RET(linear(c, true, Lout, d.Mv, eo, nullptr, s));
    }
  }
  return WAM_OK;
}

// Attach block i's LoRA A factor (action expert) to a linear layer.
void lora(wam_ctx* c, Lin& L, int i, int local, const CUtensorMap* map, const GemmPlan* plan) {
  if (c->d.r == 0) return;
  L.map_la = map;
  L.la = matp(c, blk(c->ea, i, local));
  L.plan_u = plan;
}

// ---- persistent action-block path
ActionBlockArgs ab_base(wam_ctx* c, const ActionIo* io) {
  const Dims& d = c->d;
  ActionBlockArgs a{};
  a.Ma = d.Ma;
  a.La = d.La;
  a.H = d.H;
  a.A = d.A;
  a.da = d.da;
  a.Lk = d.Lv + d.La;
  a.cache_len = d.Ltot;
  a.cache_off = d.Lv;
  a.B = d.B;
  a.x_a = c->x_a;
  a.ss = c->ab_ss;
  a.rope_cos = c->rope_cos;
  a.rope_sin = c->rope_sin;
  a.aio = io;
  a.ws = c->ab_ws;
  a.ws_half = c->ab_ws_half;
  a.ws_attn = c->ab_ws_attn;
  a.cnt = c->ab_cnt;
  a.cnt_attn = c->ab_cnt_attn;
  a.status = c->status;
  a.at.splits = c->ab_splits;
  a.at.keys = c->ab_keys;
  return a;
}

ActionGemmPhase ab_gemm(int map_w, int z, int n_out, int K, int ks, int bsrc, int map_b, int epi, const float* bias,
                        int dep) {
  ActionGemmPhase g{};
  g.map_w = map_w;
  g.z = z;
  g.n_out = n_out;
  g.K = K;
  g.ks = ks;
  g.bsrc = bsrc;
  g.map_b = map_b;
  g.epi = epi;
  g.bias = bias;
  g.dep = dep;
  g.ss_in = -1;
  g.ss_out = -1;
  g.war_phase = -1;
  return g;
}

// P^a_i: norm1 (AdaLN of block i) + merged QKV + QK-norm + RoPE + K/V publish.
ActionGemmPhase ab_qkv(wam_ctx* c, int i) {
  const Dims& d = c->d;
  const ExpertIdx& x = c->ea;
  const float* mod = c->mod_a + (size_t)i * 6 * d.da;
  ActionGemmPhase g = ab_gemm(0, i, 3 * d.A, d.da, c->ab_ks_qkv, kBNorm, 0, kEpiQkv, vecp(c, blk(x, i, kQkvB)), kDepAll);
  g.ss_in = 1;  // x_a's row sums from the FFN-down (or in-projection) tiles
  g.nscale = mod + d.da;
  g.nshift = mod;
  g.gq = vecp(c, blk(x, i, kQnG));
  g.gk = vecp(c, blk(x, i, kKnG));
  g.q_out = reinterpret_cast<__nv_bfloat16*>(c->q_a);
  g.k_cache = reinterpret_cast<__nv_bfloat16*>(kcache(c, i));
  g.v_cache = reinterpret_cast<__nv_bfloat16*>(vcache(c, i));
  return g;
}

wam_status ab_launch(wam_ctx* c, const ActionBlockArgs& a, int ctas, cudaStream_t s) {
  c->launches++;
  c->cur_cls = WAM_PROF_ACTION_BLOCK;
  ProfScope ps(c, s);
  CK(launch_action_block(c->ab_maps, a, ctas, s));
  return WAM_OK;
}

// One Euler step on the persistent path: [in-proj, P^a_0], then for every
// block i: wait(e_i) -> [Attn^a_i, R^a_i, P^a_{i+1} | output map + Euler].
wam_status enqueue_action_step_blocks(wam_ctx* c, cudaStream_t s, const ActionIo* io, int j,
                                      const cudaEvent_t* ev_wait, bool record_used) {
  const Dims& d = c->d;
  const ExpertIdx& x = c->ea;
  c->cur_cls = WAM_PROF_ACTION_TEMB;
  RET(temb(c, false, &io->sched[j], s));
  // launches that may run beside the video expert take the SMs it leaves free
  const int ctas = ev_wait ? c->ab_ctas_overlap : c->ab_ctas;
  {
    ActionBlockArgs a = ab_base(c, io);
    ActionGemmPhase in = ab_gemm(4, 0, d.da, d.Kin, c->ab_ks_in, kBTma, 8, kEpiStoreF32, vecp(c, x.inb), kDepNone);
    in.out_f32 = c->x_a;
    in.ld_out = d.da;
    in.ss_out = 1;
    a.g[a.n_gemm++] = in;
    a.g[a.n_gemm++] = ab_qkv(c, 0);
    RET(ab_launch(c, a, ctas, s));
  }
  for (int i = 0; i < d.N; ++i) {
    const float* mod = c->mod_a + (size_t)i * 6 * d.da;
    if (ev_wait) CK(cudaStreamWaitEvent(s, ev_wait[i], 0));
    trace_mark(c, s, WAM_TRACE_ACTION_ATTN, i);
    ActionBlockArgs a = ab_base(c, io);
    a.has_attn = 1;
    a.at.zk0 = (2 * i) * d.B * d.H;
    a.at.zv0 = (2 * i + 1) * d.B * d.H;
    // out-projection: B = the attention output, combined from its splits
    ActionGemmPhase o = ab_gemm(1, i, d.da, d.A, c->ab_ks_o, kBAttn, 0, kEpiGateRes, vecp(c, blk(x, i, kOB)), kDepHeads);
    o.gate = mod + 2 * d.da;
    o.out_f32 = c->x_a;
    o.ld_out = d.da;
    o.ss_out = 0;
    a.g[a.n_gemm++] = o;
    ActionGemmPhase f1 = ab_gemm(2, i, d.Fa, d.da, c->ab_ks_f1, kBNorm, 0, kEpiGelu, vecp(c, blk(x, i, kF1B)), kDepAll);
    f1.ss_in = 0;
    f1.nscale = mod + 4 * d.da;
    f1.nshift = mod + 3 * d.da;
    f1.out_act = reinterpret_cast<__nv_bfloat16*>(c->f_a);
    f1.ld_out = d.lf;
    a.g[a.n_gemm++] = f1;
    ActionGemmPhase f2 = ab_gemm(3, i, d.da, d.Fa, c->ab_ks_f2, kBTma, 7, kEpiGateRes, vecp(c, blk(x, i, kF2B)),
                                 kDepKRange);
    f2.gate = mod + 5 * d.da;
    f2.out_f32 = c->x_a;
    f2.ld_out = d.da;
    f2.ss_out = 1;
    f2.war_phase = 1;  // FFN-up's operand reads x_a: every CTA has built it before x_a changes
    a.g[a.n_gemm++] = f2;
    if (i + 1 < d.N) {
      a.g[a.n_gemm++] = ab_qkv(c, i + 1);
    } else {
      ActionGemmPhase out = ab_gemm(5, 0, d.Pa, d.da, c->ab_ks_out, kBNorm, 0, kEpiEuler, vecp(c, x.outb), kDepAll);
      out.ss_in = 1;
      out.ngain = vecp(c, x.fng);
      out.out_f32 = c->a_state;
      out.ld_out = d.Pa;
      out.step = j;
      out.a_next = reinterpret_cast<__nv_bfloat16*>(c->a_in);
      out.a_next_ld = d.Kin;
      a.g[a.n_gemm++] = out;
    }
    RET(ab_launch(c, a, ctas, s));
    trace_mark(c, s, WAM_TRACE_ACTION_END, i);
    if (record_used) CK(cudaEventRecord(c->ev_used[i], s));
  }
  return WAM_OK;
}

// One Euler step j of the action expert: P^a_i -> wait(e_i) -> Attn^a_i -> R^a_i.
wam_status enqueue_action_step(wam_ctx* c, cudaStream_t s, const ActionIo* io, int j, const cudaEvent_t* ev_wait,
                               bool record_used) {
  if (c->ab_on) return enqueue_action_step_blocks(c, s, io, j, ev_wait, record_used);
  const Dims& d = c->d;
  const ExpertIdx& x = c->ea;
  // a step that waits on the video blocks runs beside them: its attention
  // takes little shared memory per CTA so the video GEMMs keep their SMs
  c->attn_spread = ev_wait == nullptr;
  // GEMM plans by step index alone (the same in every schedule): the first
  // step may run beside the video expert, later ones run alone
  const bool later = j > 0;
  // The joint attention of a step j >= 1 reads the video rows of its keys
  // before its dependent-launch wait once kv_flag says they are complete.
  // The flag is 0 when a sequence of steps begins (zero at allocation, and
  // every sequence that may set it ends with a memset clearing it, after
  // which every later kernel on these streams starts; see clear_kv_flag).
  // Step 1's first kernel sets it once its own wait has returned, i.e. once
  // step 0 -- whose attention waited for every video block -- is complete.
  // (A memset at the start of step 0 instead put a full dependency on the
  // action stream of the captured CEWP chunk: 3.57 -> 3.75 ms.)
  if (j == 1) c->kv_flag_clean = false;
  c->attn_prefetch = later;
  const GemmPlan* pq = later ? &c->p_a_qkv_l : &c->p_a_qkv;
  const GemmPlan* po = later ? &c->p_a_o_l : &c->p_a_o;
  const GemmPlan* p1 = later ? &c->p_a_f1_l : &c->p_a_f1;
  const GemmPlan* p2 = later ? &c->p_a_f2_l : &c->p_a_f2;
  c->cur_cls = WAM_PROF_ACTION_TEMB;
  RET(temb(c, false, &io->sched[j], s, j == 1 ? c->kv_flag : nullptr));
  c->cur_cls = WAM_PROF_ACTION_IO;
  {
    Lin L{&c->m_w_in, &c->m_ain, matp(c, x.inw), c->a_state, d.da, d.bf16 ? d.Kin : d.Pa, 0, &c->p_a_in};
    RET(linear(c, false, L, d.Ma, epi_base(kEpiStoreF32, vecp(c, x.inb), c->x_a, nullptr, d.da), nullptr, s));
  }
  for (int i = 0; i < d.N; ++i) {
    const float* mod = c->mod_a + (size_t)i * 6 * d.da;
    Lin Lq{&c->m_w_qkv_a, &c->m_ha, matp(c, blk(x, i, kQkvW)), c->h_a, 3 * d.A, d.da, i, pq, d.lh};
    lora(c, Lq, i, kQkvLa, &c->m_la_qkv, &c->p_u_qkv);
    RET(norm_linear(c, Lq, epi_qkv(c, false, i), mod + d.da, mod, nullptr, WAM_PROF_ACTION_QKV, s));
    if (ev_wait) CK(cudaStreamWaitEvent(s, ev_wait[i], 0));
    trace_mark(c, s, WAM_TRACE_ACTION_ATTN, i);
    c->cur_cls = WAM_PROF_ACTION_ATTN;
    RET(attention(c, false, i, s));
    if (record_used) CK(cudaEventRecord(c->ev_used[i], s));
    c->cur_cls = WAM_PROF_ACTION_OPROJ;
    EpiArgs eo = epi_base(kEpiGateRes, vecp(c, blk(x, i, kOB)), c->x_a, nullptr, d.da);
    eo.gate = mod + 2 * d.da;
    Lin Lo{&c->m_w_o_a, &c->m_oa, matp(c, blk(x, i, kOW)), c->o_a, d.da, d.A, i, po, d.lo};
    lora(c, Lo, i, kOLa, &c->m_la_o, &c->p_u_o);
    RET(linear(c, false, Lo, d.Ma, eo, nullptr, s));
    Lin L1{&c->m_w_f1_a, &c->m_ha, matp(c, blk(x, i, kF1W)), c->h_a, d.Fa, d.da, i, p1, d.lh};
    lora(c, L1, i, kF1La, &c->m_la_f1, &c->p_u_f1);
    RET(norm_linear(c, L1, epi_base(kEpiGelu, vecp(c, blk(x, i, kF1B)), nullptr, c->f_a, d.lf), mod + 4 * d.da,
                    mod + 3 * d.da, nullptr, WAM_PROF_ACTION_FFN_UP, s));
    c->cur_cls = WAM_PROF_ACTION_FFN_DOWN;
    EpiArgs e2 = epi_base(kEpiGateRes, vecp(c, blk(x, i, kF2B)), c->x_a, nullptr, d.da);
    e2.gate = mod + 5 * d.da;
    Lin L2{&c->m_w_f2_a, &c->m_fa, matp(c, blk(x, i, kF2W)), c->f_a, d.da, d.Fa, i, p2, d.lf};
    lora(c, L2, i, kF2La, &c->m_la_f2, &c->p_u_f2);
    RET(linear(c, false, L2, d.Ma, e2, nullptr, s));
    trace_mark(c, s, WAM_TRACE_ACTION_END, i);
  }
  EpiArgs ee = epi_base(kEpiEuler, vecp(c, x.outb), c->a_state, nullptr, d.Pa);
  ee.aio = io;
  ee.step = j;
  ee.a_next = d.bf16 ? c->a_in : nullptr;
  ee.a_next_ld = d.Kin;
  Lin Lout{&c->m_w_out, &c->m_ha, matp(c, x.outw), c->h_a, d.Pa, d.da, 0, &c->p_a_out, d.lh};
  RET(norm_linear(c, Lout, ee, nullptr, nullptr, vecp(c, x.fng), WAM_PROF_ACTION_IO, s));
  return WAM_OK;
}

// kv_flag back to 0 at the end of a sequence of Euler steps (every later
// kernel on the stream starts after the memset completes).
wam_status clear_kv_flag(wam_ctx* c, cudaStream_t s) {
  CK(cudaMemsetAsync(c->kv_flag, 0, sizeof(int), s));
  c->kv_flag_clean = true;
  return WAM_OK;
}

// A whole chunk: video once, then `steps` Euler steps (or the joint one-step).
wam_status enqueue_chunk(wam_ctx* c, int steps, int mode, bool joint, cudaStream_t sv, cudaStream_t sa,
                         cudaEvent_t* ev_kv, int n_video = 0) {
  const Dims& d = c->d;
  if (!c->kv_flag_clean) RET(clear_kv_flag(c, sv));  // an earlier sequence stopped before its end
  const bool cewp = mode == WAM_SCHED_CEWP;
  cudaStream_t s_act = cewp ? sa : sv;
  if (cewp) {
    CK(cudaEventRecord(c->ev_fork, sv));
    CK(cudaStreamWaitEvent(sa, c->ev_fork, 0));
  }
  // action-side prologue (no dependence on the video expert)
  c->launches++;
  c->cur_cls = WAM_PROF_ACTION_IO;
  {
  ProfScope ps(c, s_act);
  if (joint)
    CK(launch_noise_action(c->aio_chunk, c->a_state, d.bf16 ? c->a_in : nullptr, d.bf16, d.Ma, d.Pa, d.Kin, s_act));
  else
    CK(launch_init_action(c->aio_chunk, c->a_state, d.bf16 ? c->a_in : nullptr, d.bf16, d.Ma, d.Pa, d.Kin, s_act));
  }
  if (cewp) {
    // The experts need not be enqueued interleaved block by block: the two
    // streams run concurrently, and the per-block events order Attn^a_i after P^v_i.
    RET(enqueue_video(c, sv, c->vio_chunk, joint, ev_kv, false, n_video));
    for (int j = 0; j < steps; ++j) {
      c->trace_step = j;
      RET(enqueue_action_step(c, sa, c->aio_chunk, j, j == 0 ? ev_kv : nullptr, false));
    }
  } else {
    RET(enqueue_video(c, sv, c->vio_chunk, joint, nullptr, false, n_video));
    for (int j = 0; j < steps; ++j) {
      c->trace_step = j;
      RET(enqueue_action_step(c, sv, c->aio_chunk, j, nullptr, false));
    }
  }
  c->trace_step = 0;
  c->launches++;
  {
    c->cur_cls = WAM_PROF_ACTION_IO;
    ProfScope ps(c, s_act);
    CK(launch_copy_out(c->aio_chunk, c->a_state, d.Ma * d.Pa, s_act));
  }
  if (cewp) {
    CK(cudaEventRecord(c->ev_join, sa));
    CK(cudaStreamWaitEvent(sv, c->ev_join, 0));
  }
  if (steps > 1) RET(clear_kv_flag(c, sv));
  return WAM_OK;
}

wam_status set_chunk_io(wam_ctx* c, const VideoIo& v, const ActionIo& a, cudaStream_t sv) {
  if (!c->vio_valid || memcmp(&v, &c->vio_shadow, sizeof v) != 0) {
    CK(launch_set_video_io(c->vio_chunk, v, sv));
    c->vio_shadow = v;
    c->vio_valid = true;
  }
  if (!c->aio_valid || memcmp(&a, &c->aio_shadow, sizeof a) != 0) {
    CK(launch_set_action_io(c->aio_chunk, a, sv));
    c->aio_shadow = a;
    c->aio_valid = true;
  }
  return WAM_OK;
}

// Graph key of a chunk: Euler steps, video passes, schedule, joint variant.
long long chunk_key(int steps, int n_video, int mode, bool joint) {
  return ((long long)steps << 24) | ((long long)n_video << 16) | (mode << 1) | (joint ? 1 : 0);
}

wam_status run_chunk(wam_ctx* c, int steps, int mode, int use_graph, bool joint, cudaStream_t sv, cudaStream_t sa,
                     int n_video = 0) {
  const long long key = chunk_key(steps, n_video, mode, joint);
  if (!use_graph) {
    c->launches = 0;
    RET(enqueue_chunk(c, steps, mode, joint, sv, mode == WAM_SCHED_CEWP ? sa : sv, c->ev_kv.data(), n_video));
    c->launch_counts[key] = c->launches;
  } else {
    auto it = c->graphs.find(key);
    if (it == c->graphs.end()) {
      cudaGraph_t graph = nullptr;
      c->launches = 0;
      CK(cudaStreamBeginCapture(c->cap_v, cudaStreamCaptureModeThreadLocal));
      wam_status st = enqueue_chunk(c, steps, mode, joint, c->cap_v, c->cap_a, c->ev_kv_cap.data(), n_video);
      cudaError_t ce = cudaStreamEndCapture(c->cap_v, &graph);
      if (st != WAM_OK) {
        if (graph) cudaGraphDestroy(graph);
        return st;
      }
      CK(ce);
      cudaGraphExec_t exec = nullptr;
      cudaError_t ie = cudaGraphInstantiate(&exec, graph, 0);
      cudaGraphDestroy(graph);
      CK(ie);
      it = c->graphs.emplace(key, exec).first;
      c->launch_counts[key] = c->launches;
    }
    CK(cudaGraphLaunch(it->second, sv));
  }
  if (mode == WAM_SCHED_CEWP && sa != sv) {
    CK(cudaEventRecord(c->ev_post, sv));
    CK(cudaStreamWaitEvent(sa, c->ev_post, 0));
  }
  return WAM_OK;
}

bool valid_schedule(const float* t, int S) {
  for (int j = 0; j <= S; ++j)
    if (!(t[j] >= 0.f && t[j] <= 1.f)) return false;
  for (int j = 0; j < S; ++j)
    if (!(t[j] > t[j + 1])) return false;
  return true;
}

template <typename T>
wam_status dalloc(wam_ctx* c, T** p, size_t bytes) {
  if (bytes == 0) bytes = 256;
  if (c->mem_limit && c->mem_used + bytes > c->mem_limit)
    return fail(c, WAM_ERR_OOM, "allocation of %zu bytes exceeds the context's device memory limit (%zu of %zu used)",
                bytes, c->mem_used, c->mem_limit);
  cudaError_t e = cudaMalloc((void**)p, bytes);
  if (e == cudaErrorMemoryAllocation) {
    cudaGetLastError();
    return fail(c, WAM_ERR_OOM, "cudaMalloc(%zu) failed: out of device memory", bytes);
  }
  CK(e);
  c->mem_used += bytes;
  CK(cudaMemset(*p, 0, bytes));
  return WAM_OK;
}

bool check_cfg(const wam_config* g, std::string* why) {
  auto bad = [&](const char* m) {
    *why = m;
    return false;
  };
  if (g->n_blocks < 1 || g->d_video < 8 || g->d_action < 8 || g->n_heads < 1 || g->head_dim < 2) return bad("sizes must be positive");
  if (g->l_video < 1 || g->l_action < 1 || g->l_cond < 0 || g->batch < 1 || g->action_dim < 1) return bad("token counts");
  if (g->head_dim % 2) return bad("head_dim must be even");
  if (g->d_video % 8 || g->d_action % 8 || g->ffn_video % 8 || g->ffn_action % 8) return bad("widths must be multiples of 8");
  // the norm / modulation prologue keeps a whole row in one warp's registers
  if (g->d_video > 1536 || g->d_action > 1536) return bad("expert widths above 1536 are not supported");
  if (g->video_has_output && g->video_patch_dim <= 0) return bad("a video output needs patch input");
  if (g->video_patch_dim > 0 && g->l_cond != 0) return bad("patch input takes no conditioning tokens");
  if (g->lora_rank < 0) return bad("lora_rank");
  if (g->dtype == WAM_BF16) {
    const int A = g->n_heads * g->head_dim;
    if (g->head_dim != 64) return bad("bf16 path needs head_dim 64");
    if (g->d_video % 64 || g->d_action % 64 || g->ffn_video % 128 || g->ffn_action % 64 || A % 128)
      return bad("bf16 path needs widths in multiples of 64 (ffn_video, attention width: 128)");
    if (g->video_patch_dim % 64) return bad("bf16 path needs video_patch_dim multiple of 64");
    if (g->batch * g->l_action > 256) return bad("bf16 path supports at most 256 action tokens per chunk");
    if (g->l_action > 64) return bad("bf16 path supports at most 64 action tokens per sample");
    if (g->lora_rank > 0 && g->lora_rank % 64) return bad("lora_rank must be a multiple of 64");
  } else if (g->dtype == WAM_FP32) {
    if (g->head_dim > 64 || (g->head_dim != 16 && g->head_dim != 32 && g->head_dim != 64))
      return bad("fp32 path supports head_dim 16, 32, 64");
    if (g->d_video % 4 || g->d_action % 4) return bad("fp32 widths must be multiples of 4");
  } else {
    return bad("dtype");
  }
  return true;
}

}  // namespace

// ===================================================================== ABI ==
extern "C" {

wam_status wam_preset(int k, wam_config* o) {
  if (!o) return WAM_ERR_INVALID_ARG;
  wam_config g{};
  g.action_dim = 30;
  g.batch = 1;
  g.lora_scale = 1.0f;
  switch (k) {
    case 1:
      g.n_blocks = 2; g.d_video = 64; g.d_action = 64; g.n_heads = 4; g.head_dim = 16;
      g.ffn_video = 256; g.ffn_action = 256; g.l_cond = 0; g.l_video = 64; g.l_action = 16;
      g.dtype = WAM_FP32;
      break;
    case 2:
    case 3:
    case 4:
      g.n_blocks = 28; g.d_video = 1536; g.d_action = 768; g.n_heads = 24; g.head_dim = 64;
      g.ffn_video = 6144; g.ffn_action = 3072; g.l_cond = 64; g.l_video = 1024; g.l_action = 32;
      g.dtype = WAM_BF16;
      if (k == 4) {
        g.l_video = 2048;
        g.batch = 8;
      }
      break;
    case 5:
      g.n_blocks = 30; g.d_video = 1536; g.d_action = 1536; g.n_heads = 24; g.head_dim = 64;
      g.ffn_video = 6144; g.ffn_action = 6144; g.l_cond = 0; g.l_video = 1024; g.l_action = 16;
      g.video_patch_dim = 192; g.lora_rank = 128; g.video_has_output = 1; g.dtype = WAM_BF16;
      break;
    default:
      return WAM_ERR_INVALID_ARG;
  }
  *o = g;
  return WAM_OK;
}

const char* wam_status_str(wam_status s) {
  switch (s) {
    case WAM_OK: return "ok";
    case WAM_ERR_INVALID_ARG: return "invalid argument";
    case WAM_ERR_UNSUPPORTED: return "unsupported";
    case WAM_ERR_OOM: return "out of device memory";
    case WAM_ERR_CUDA: return "CUDA error";
    case WAM_ERR_TIMEOUT: return "device wait timed out";
    case WAM_ERR_STATE: return "invalid call order";
  }
  return "unknown status";
}

const char* wam_last_error(wam_ctx* c) { return c ? c->last_error.c_str() : ""; }

void wam_destroy(wam_ctx* c) {
  if (!c) return;
  cudaSetDevice(c->device);
  cudaDeviceSynchronize();
  for (auto& kv : c->graphs) cudaGraphExecDestroy(kv.second);
  for (auto* v : {&c->ev_kv, &c->ev_kv_cap, &c->ev_used})
    for (auto e : *v)
      if (e) cudaEventDestroy(e);
  for (auto e : {c->ev_fork, c->ev_join, c->ev_pre, c->ev_post})
    if (e) cudaEventDestroy(e);
  for (auto e : c->prof_pool) cudaEventDestroy(e);
  for (auto e : c->trace_pool) cudaEventDestroy(e);
  if (c->cap_v) cudaStreamDestroy(c->cap_v);
  if (c->cap_a) cudaStreamDestroy(c->cap_a);
  void* bufs[] = {c->wmat, c->wvec, c->x_v, c->x_a, c->a_state, c->x_sigma, c->h_v, c->q_v, c->o_v, c->f_v,
                  c->x_vin, c->h_a, c->q_a, c->o_a, c->f_a, c->a_in, c->qkv_tmp_v, c->qkv_tmp_a, c->kv,
                  c->mod_v, c->mod_a, c->temb_v, c->temb_a, c->rope_cos, c->rope_sin, c->ws_gemm, c->tk_gemm, c->ws_gemm_v, c->tk_gemm_v, c->zero_r,
                  c->ws_attn, c->tk_attn, c->status, c->vio_chunk, c->vio_eager, c->aio_chunk, c->aio_eager,
                  c->h_video, c->h_cond, c->h_noise, c->h_out, c->j_vout, c->j_aout, c->ab_ws, c->ab_ws_attn,
                  c->ab_ss, c->ab_cnt, c->ab_cnt_attn, c->td_at, c->td_as, c->td_a0, c->td_fs, c->td_fe,
                  c->aio_tacd};
  for (void* p : bufs)
    if (p) cudaFree(p);
  delete c;
}

wam_status wam_init(const wam_config* cfg, uint64_t seed, wam_ctx** out) {
  if (!cfg || !out) return WAM_ERR_INVALID_ARG;
  std::string why;
  if (!check_cfg(cfg, &why)) return WAM_ERR_INVALID_ARG;
  // on any failure below, wam_destroy releases what was created so far
  std::unique_ptr<wam_ctx, void (*)(wam_ctx*)> holder(new wam_ctx(), wam_destroy);
  wam_ctx* c = holder.get();
  c->cfg = *cfg;
  if (const char* v = getenv("WAM_DEVICE_MEMORY_LIMIT")) c->mem_limit = strtoull(v, nullptr, 10);
  CK(cudaGetDevice(&c->device));
  CK(prepare_tc_gemm());
  CK(prepare_attention_tc());
  CK(prepare_attention_bf16());
  CK(prepare_attention_joint());
  Dims& d = c->d;
  d.N = cfg->n_blocks; d.dv = cfg->d_video; d.da = cfg->d_action; d.H = cfg->n_heads; d.Dh = cfg->head_dim;
  d.A = d.H * d.Dh; d.Fv = cfg->ffn_video; d.Fa = cfg->ffn_action; d.Lc = cfg->l_cond; d.Lvid = cfg->l_video;
  d.Lv = d.Lc + d.Lvid; d.La = cfg->l_action; d.Pa = cfg->action_dim; d.Pv = cfg->video_patch_dim;
  d.B = cfg->batch; d.r = cfg->lora_rank; d.Ltot = d.Lv + d.La; d.Mv = d.B * d.Lv; d.Ma = d.B * d.La;
  d.bf16 = cfg->dtype == WAM_BF16;
  d.Kin = d.bf16 ? (d.Pa + 63) / 64 * 64 : d.Pa;
  d.lh = d.da + d.r;
  d.lo = d.A + d.r;
  d.lf = d.Fa + d.r;
  c->esz = d.bf16 ? 2 : 4;

  add_expert(c, true);
  add_expert(c, false);
  layout_params(c);

  RET(dalloc(c, &c->wmat, c->wmat_elems * c->esz));
  RET(dalloc(c, &c->wvec, c->wvec_elems * sizeof(float)));
  for (size_t p = 0; p < c->params.size(); ++p) {
    const PEntry& e = c->params[p];
    void* dst = e.matrix ? matp(c, (int)p) : (void*)vecp(c, (int)p);
    CK(launch_gen_param(seed, p, e.count(), 0.02, e.ones, d.bf16, dst, e.matrix && d.bf16, e.cols,
                        e.matrix ? e.ld : e.cols, 0));
  }

  const size_t ae = c->esz;
  RET(dalloc(c, &c->x_v, (size_t)d.Mv * d.dv * 4));
  RET(dalloc(c, &c->h_v, (size_t)d.Mv * d.dv * ae));
  RET(dalloc(c, &c->q_v, (size_t)d.Mv * d.A * ae));
  RET(dalloc(c, &c->o_v, (size_t)d.Mv * d.A * ae));
  RET(dalloc(c, &c->f_v, (size_t)d.Mv * d.Fv * ae));
  RET(dalloc(c, &c->x_a, (size_t)d.Ma * d.da * 4));
  RET(dalloc(c, &c->h_a, (size_t)d.Ma * d.lh * ae));
  RET(dalloc(c, &c->q_a, (size_t)d.Ma * d.A * ae));
  RET(dalloc(c, &c->o_a, (size_t)d.Ma * d.lo * ae));
  RET(dalloc(c, &c->f_a, (size_t)d.Ma * d.lf * ae));
  RET(dalloc(c, &c->zero_r, (size_t)std::max(d.r, 1) * 4));
  RET(dalloc(c, &c->a_state, (size_t)d.Ma * d.Pa * 4));
  RET(dalloc(c, &c->a_in, (size_t)d.Ma * d.Kin * ae));
  if (d.Pv > 0) {
    RET(dalloc(c, &c->x_sigma, (size_t)d.Mv * d.Pv * 4));
    RET(dalloc(c, &c->x_vin, (size_t)d.Mv * d.Pv * ae));
  }
  if (!d.bf16) {
    RET(dalloc(c, &c->qkv_tmp_v, (size_t)d.Mv * 3 * d.A * 4));
    RET(dalloc(c, &c->qkv_tmp_a, (size_t)d.Ma * 3 * d.A * 4));
  }
  RET(dalloc(c, &c->kv, (size_t)2 * d.N * d.B * d.H * d.Ltot * d.Dh * ae));
  RET(dalloc(c, &c->mod_v, (size_t)d.N * 6 * d.dv * 4));
  RET(dalloc(c, &c->mod_a, (size_t)d.N * 6 * d.da * 4));
  RET(dalloc(c, &c->temb_v, (size_t)(256 + 2 * d.dv) * 4));
  RET(dalloc(c, &c->temb_a, (size_t)(256 + 2 * d.da) * 4));
  RET(dalloc(c, &c->rope_cos, (size_t)d.Ltot * d.Dh / 2 * 4));
  RET(dalloc(c, &c->rope_sin, (size_t)d.Ltot * d.Dh / 2 * 4));
  RET(dalloc(c, &c->status, 256));
  RET(dalloc(c, &c->vio_chunk, sizeof(VideoIo)));
  RET(dalloc(c, &c->vio_eager, sizeof(VideoIo)));
  RET(dalloc(c, &c->aio_chunk, sizeof(ActionIo)));
  RET(dalloc(c, &c->aio_eager, sizeof(ActionIo)));
  RET(dalloc(c, &c->kv_flag, sizeof(int)));  // (zeroed)
  CK(launch_rope_table(c->rope_cos, c->rope_sin, d.Ltot, d.Dh, 0));

  // GEMM plans (bf16 path) and workspaces
  size_t ws = 0, ws_v = 0;
  int tiles = 1, tiles_v = 1;
  if (d.bf16) {
    // Video GEMMs (tokens on TMEM lanes): stream-K over a persistent grid, so
    // every CTA gets the same share of k-blocks whatever the tile count.  QKV
    // and FFN-up take 256-feature tiles (half the operand traffic per flop of
    // 128).  Out-proj / FFN-down (d-wide outputs, gate-residual epilogue) take
    // 256 only when that still leaves two tiles per CTA: with fewer, the
    // split-tile reduction and the last tile's residual epilogue cost more
    // than the faster MMA saves (1088 tokens: 18.9 -> 27.4 us out-proj).  The
    // video GEMMs leave about a quarter of
    // the SMs to the action stream that runs beside them under CEWP (108 of
    // 148 measured best on the config-2 chunk; WAM_VIDEO_GEMM_CTAS overrides
    // the count).  The grid is the same in every schedule: the k-range
    // split points, and so every rounding, do not depend on the schedule.
    int nsm = 148;
    CK(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, c->device));
    int vctas = std::max(1, nsm * 73 / 100);
    if (const char* v = getenv("WAM_VIDEO_GEMM_CTAS")) {
      const int n = atoi(v);
      if (n > 0) vctas = std::min(n, nsm);
    }
    // With at most two tiles per CTA, take the largest grid <= vctas that
    // the tile count divides: whole tiles per CTA, no split-tile reduction
    // in the short tail (QKV at 1088 tokens: 162 tiles on 81 CTAs instead of
    // 1.5 tiles on each of 108; chunk 4.33 -> 4.15 ms).  With more tiles per
    // CTA the split overhead is small and all vctas CTAs are kept.
    // WAM_VIDEO_SPLIT_FREE=0 turns the rule off (always vctas CTAs, stream-K).
    const char* sfv = getenv("WAM_VIDEO_SPLIT_FREE");
    const bool split_free = !(sfv && sfv[0] == '0');
    // CTA pairs (2-SM MMA, M = 256 over two SMs; WAM_VIDEO_PAIR=1): each SM
    // stages its own 128 token rows and half of the 256 weight rows of a
    // tile, half the operand bytes per flop of a 1-SM 128 x 256 tile.  Off by
    // default: the 1-SM 256-wide main loop already runs at the tensor-core
    // rate (0.38 us per 64-deep k-block at 1088 tokens, both forms), and the
    // pairs' longer split-tile tails made them slower (FFN-down 41 vs 30 us).
    const char* pv = getenv("WAM_VIDEO_PAIR");
    const bool pair = pv && pv[0] == '1' && d.dv % 256 == 0 && (3 * d.A) % 256 == 0 && d.Fv % 256 == 0;
    auto grid = [&](int n_out, int bn, bool pr) {
      const int unit_rows = pr ? 256 : 128, units = pr ? vctas / 2 : vctas;
      const int tiles = ((d.Mv + unit_rows - 1) / unit_rows) * ((n_out + bn - 1) / bn);
      const int k = (tiles + units - 1) / units;  // tiles per unit
      // whole tiles per unit, unless that leaves a quarter of the units idle
      const bool whole = split_free && k <= 2 && tiles % k == 0 && 4 * (tiles / k) >= 3 * units;
      return (whole ? tiles / k : units) * (pr ? 2 : 1);
    };
    const int bn_res = ((d.Mv + 127) / 128) * (d.dv / 256) >= 2 * vctas ? 256 : 128;
    // WAM_VIDEO_OPROJ_BN / WAM_VIDEO_FFN2_BN (128 or 256) override the tile
    // width of the two gate-residual GEMMs
    auto bn_env = [&](const char* name, int dflt) {
      const char* v = getenv(name);
      const int n = v ? atoi(v) : 0;
      return (n == 128 || n == 256) && d.dv % n == 0 ? n : dflt;
    };
    const int bn_o = bn_env("WAM_VIDEO_OPROJ_BN", bn_res), bn_f2 = bn_env("WAM_VIDEO_FFN2_BN", bn_res);
    if (pair) {
      c->p_v_qkv = {256, 1, grid(3 * d.A, 256, true), true};
      c->p_v_o = {256, 1, grid(d.dv, 256, true), true};
      c->p_v_f1 = {256, 1, grid(d.Fv, 256, true), true};
      c->p_v_f2 = {256, 1, grid(d.dv, 256, true), true};
    } else {
      // QKV on 256- or 192-wide tiles, whichever puts whole tiles on more
      // CTAs (1088 tokens: 162 tiles of 256 on 81 CTAs, 216 tiles of 192 on
      // 108 -- the per-k-block rate is the same, so the MMA time drops by a
      // quarter); the QK-norm epilogue needs the tile width to divide the
      // attention width.  WAM_VIDEO_QKV_BN (192 or 256) overrides.
      auto whole_units = [&](int n_out, int bn) {
        const int tiles = ((d.Mv + 127) / 128) * ((n_out + bn - 1) / bn);
        const int k = (tiles + vctas - 1) / vctas;
        return (split_free && k <= 2 && tiles % k == 0) ? tiles / k : 0;
      };
      int bn_qkv = 256;
      if (d.A % 192 == 0 && whole_units(3 * d.A, 192) > whole_units(3 * d.A, 256)) bn_qkv = 192;
      if (const char* v = getenv("WAM_VIDEO_QKV_BN")) {
        const int n = atoi(v);
        if ((n == 192 || n == 256) && d.A % n == 0) bn_qkv = n;
      }
      c->p_v_qkv = {bn_qkv, 1, grid(3 * d.A, bn_qkv, false)};
      c->p_v_o = {bn_o, 1, grid(d.dv, bn_o, false)};
      c->p_v_f1 = {256, 1, grid(d.Fv, 256, false)};
      c->p_v_f2 = {bn_f2, 1, grid(d.dv, bn_f2, false)};
      // Cluster split for the d-wide gate-residual GEMMs when their 256-wide
      // tiles number about half the grid and each half of the k-range is at
      // least 24 k-blocks deep: each tile's k-range is split between the two
      // CTAs of a cluster, which finish it in column halves (the partials
      // crossing in shared memory, ~3 us).  At 1088 tokens FFN-down (96
      // k-blocks): 54 tiles on 108 CTAs, 36.9 -> 26.1 us per launch alone,
      // config-2 chunk 4.12 -> 3.91 ms.  The out-projection (24 k-blocks) is
      // left on 128-wide whole tiles: split, it measured 1.7 us slower per
      // launch in the chunk.  WAM_VIDEO_CSPLIT=0 (or a tile-width override)
      // keeps the rule above.
      const char* csv = getenv("WAM_VIDEO_CSPLIT");
      const bool csplit_ok = !(csv && csv[0] == '0');
      auto csplit_plan = [&](GemmPlan* p, int n_out, int K, const char* bn_var) {
        const int tiles = ((d.Mv + 127) / 128) * (n_out / 256);
        if (!csplit_ok || getenv(bn_var) || n_out % 256 || 2 * tiles > nsm || 4 * (2 * tiles) < 3 * vctas ||
            K / 64 < 48)
          return;
        *p = GemmPlan{256, 1, 2 * tiles, false, true};
      };
      csplit_plan(&c->p_v_o, d.dv, d.A, "WAM_VIDEO_OPROJ_BN");
      csplit_plan(&c->p_v_f2, d.dv, d.Fv, "WAM_VIDEO_FFN2_BN");
    }
    c->p_v_in = {128, 1, grid(d.dv, 128, false)};
    c->p_v_out = {64, 1, grid(d.Pv > 0 ? d.Pv : 64, 64, false)};
    const int bn_a = d.Ma <= 32 ? 32 : (d.Ma <= 64 ? 64 : (d.Ma <= 128 ? 128 : 256));
    // Opt-in (WAM_FUSE_NORM=1): every CTA of the fused GEMM re-reads all of
    // x_a for the row norms, and on the config-2/3 chunks that measured slower
    // under CEWP (4.45 / 21.5 ms) than the separate norm kernel (4.38 / 20.4).
    const char* fv = getenv("WAM_FUSE_NORM");
    c->fuse_norm_a = fv && fv[0] == '1' && bn_a <= 64 && d.da <= 1024 && d.da % 64 == 0 && d.r == 0;
    const bool fn = c->fuse_norm_a;
    // Opt-in (WAM_VIDEO_FUSED_NORM=1): the video QKV / FFN-up GEMMs compute
    // their A operand (the block's RMSNorm + AdaLN modulation of x_v) in their
    // own prologue instead of a separate norm launch.  Off by default: in the
    // captured chunk the norm kernel starts early (dependent launch) and costs
    // ~2-3 us on the critical path, while the prologue runs the 1088 rows on
    // only four warps per CTA before the first MMA (config-2 chunk 4.77 ms
    // fused against 4.12 ms).
    const char* fvv = getenv("WAM_VIDEO_FUSED_NORM");
    c->fuse_norm_v = fvv && fvv[0] == '1' && d.dv % 4 == 0 && d.dv <= kRowNormMax;
    // CTAs per action GEMM (tiles x splits, about): the weight stream spread
    // over this many SMs; WAM_ACTION_CTAS overrides.
    int actas = nsm;
    if (const char* v = getenv("WAM_ACTION_CTAS")) {
      const int n = atoi(v);
      if (n > 0) actas = n;
    }
    // Split action GEMMs sum their pieces in a cluster's shared memory;
    // WAM_ACTION_CRED=0 keeps the same splits but sums through global
    // partials (the stream-K tickets).
    const char* crv = getenv("WAM_ACTION_CRED");
    const bool cred_on = !(crv && crv[0] == '0');
    c->p_a_in = plan_swap(d.da, d.Ma, d.Kin, bn_a, false, actas);
    // The first Euler step runs beside the video expert: its GEMMs keep the
    // stream-K plans (the cluster plans below took SMs from the video stream,
    // config-2 chunk 3.54 -> 3.80 ms).  Later steps run alone and use them.
    c->p_a_qkv = plan_swap(3 * d.A, d.Ma, d.da + d.r, bn_a, fn, actas);
    c->p_a_o = plan_swap(d.da, d.Ma, d.A + d.r, bn_a, false, actas);
    c->p_a_f1 = plan_swap(d.Fa, d.Ma, d.da + d.r, bn_a, fn, actas);
    c->p_a_f2 = plan_swap(d.da, d.Ma, d.Fa + d.r, bn_a, false, actas);
    // The wide action FFN-up (24 or more feature tiles) splits each tile
    // over a cluster of WAM_ACTION_WIDE_SPLITS CTAs (default 4; 0 or 1:
    // unsplit): with the pieces summed in shared memory the split pays (the
    // 10-step chunk's FFN-up 9.3 -> 5.9 us per launch at 4).  The QKV GEMM
    // (36 tiles) takes WAM_ACTION_QKV_SPLITS (default 2: 8.6 -> 7.8 us; at 4
    // its 144 CTAs in clusters did not all find SMs at once, 8.3 -> 12.1 us).
    int wide = 4, wide_qkv = 2;
    if (const char* v = getenv("WAM_ACTION_WIDE_SPLITS")) wide = atoi(v);
    if (const char* v = getenv("WAM_ACTION_QKV_SPLITS")) wide_qkv = atoi(v);
    c->p_a_qkv_l = plan_swap(3 * d.A, d.Ma, d.da + d.r, bn_a, fn, actas, wide_qkv > 1, wide_qkv);
    c->p_a_o_l = plan_swap(d.da, d.Ma, d.A + d.r, bn_a, false, actas, true);
    c->p_a_f1_l = plan_swap(d.Fa, d.Ma, d.da + d.r, bn_a, fn, actas, wide > 1, wide);
    c->p_a_f2_l = plan_swap(d.da, d.Ma, d.Fa + d.r, bn_a, false, actas, true);
    if (!cred_on) {
      c->p_a_qkv_l.cred = 0;
      c->p_a_o_l.cred = 0;
      c->p_a_f1_l.cred = 0;
      c->p_a_f2_l.cred = 0;
    }
    if (d.r > 0) {
      c->p_u_qkv = plan_swap(d.r, d.Ma, d.da, bn_a, false, actas);
      c->p_u_o = plan_swap(d.r, d.Ma, d.A, bn_a, false, actas);
      c->p_u_f1 = plan_swap(d.r, d.Ma, d.da, bn_a, false, actas);
      c->p_u_f2 = plan_swap(d.r, d.Ma, d.Fa, bn_a, false, actas);
    }
    c->p_a_out = plan_swap(d.Pa, d.Ma, d.da, bn_a, fn, actas);
    // workspace and tickets of one launch: rows_a x rows_b output, reduction K
    auto need = [](const GemmPlan& p, int rows_a, int rows_b, int K, bool swap, size_t* w, int* t) {
      TcGemm g{};
      g.rows_a = rows_a;
      g.rows_b = rows_b;
      g.K = K;
      g.bn = p.bn;
      g.splits = p.splits;
      g.swap = swap;
      g.max_ctas = p.max_ctas;
      g.pair = p.pair;
      *w = std::max(*w, tc_gemm_ws_floats(g));
      *t = std::max(*t, (int)(tc_gemm_tickets(g) / 2));
    };
    need(c->p_a_in, d.da, d.Ma, d.Kin, true, &ws, &tiles);
    need(c->p_a_qkv, 3 * d.A, d.Ma, d.da + d.r, true, &ws, &tiles);
    need(c->p_a_o, d.da, d.Ma, d.A + d.r, true, &ws, &tiles);
    need(c->p_a_f1, d.Fa, d.Ma, d.da + d.r, true, &ws, &tiles);
    need(c->p_a_f2, d.da, d.Ma, d.Fa + d.r, true, &ws, &tiles);
    need(c->p_a_qkv_l, 3 * d.A, d.Ma, d.da + d.r, true, &ws, &tiles);
    need(c->p_a_o_l, d.da, d.Ma, d.A + d.r, true, &ws, &tiles);
    need(c->p_a_f1_l, d.Fa, d.Ma, d.da + d.r, true, &ws, &tiles);
    need(c->p_a_f2_l, d.da, d.Ma, d.Fa + d.r, true, &ws, &tiles);
    if (d.r > 0) {
      need(c->p_u_qkv, d.r, d.Ma, d.da, true, &ws, &tiles);
      need(c->p_u_o, d.r, d.Ma, d.A, true, &ws, &tiles);
      need(c->p_u_f1, d.r, d.Ma, d.da, true, &ws, &tiles);
      need(c->p_u_f2, d.r, d.Ma, d.Fa, true, &ws, &tiles);
    }
    need(c->p_a_out, d.Pa, d.Ma, d.da, true, &ws, &tiles);
    need(c->p_v_qkv, d.Mv, 3 * d.A, d.dv, false, &ws_v, &tiles_v);
    need(c->p_v_o, d.Mv, d.dv, d.A, false, &ws_v, &tiles_v);
    need(c->p_v_f1, d.Mv, d.Fv, d.dv, false, &ws_v, &tiles_v);
    need(c->p_v_f2, d.Mv, d.dv, d.Fv, false, &ws_v, &tiles_v);
    if (d.Pv > 0) need(c->p_v_in, d.Mv, d.dv, d.Pv, false, &ws_v, &tiles_v);
    if (cfg->video_has_output) need(c->p_v_out, d.Mv, d.Pv, d.dv, false, &ws_v, &tiles_v);
    c->attn_splits = std::max(1, (d.Lv + d.La + 127) / 128);
    // Joint action attention on clusters of key splits (WAM_JOINT_ATTN=0:
    // the split-KV kernel with a ticket combine)
    const char* jav = getenv("WAM_JOINT_ATTN");
    if (!(jav && jav[0] == '0') && d.Dh == 64 && d.La <= 64)
      c->attn_joint_splits = attention_joint_splits(d.B * d.H, d.La, d.Lv + d.La, nsm);
  }
  RET(dalloc(c, &c->ws_gemm, ws * 4));
  RET(dalloc(c, &c->tk_gemm, (size_t)tiles * 2 * 4));
  c->tk_gemm_bytes = (size_t)tiles * 2 * 4;
  RET(dalloc(c, &c->ws_gemm_v, ws_v * 4));
  RET(dalloc(c, &c->tk_gemm_v, (size_t)tiles_v * 2 * 4));
  RET(dalloc(c, &c->na_cnt, 3 * 4));
  c->tk_gemm_v_bytes = (size_t)tiles_v * 2 * 4;
  RET(dalloc(c, &c->ws_attn, attention_ws_floats(d.B, d.H, d.Dh, d.La, c->attn_splits) * 4));
  RET(dalloc(c, &c->tk_attn, (size_t)d.B * d.H * 4));

  if (d.bf16) {
    bool ok = true;
    auto wmap = [&](CUtensorMap* m, const ExpertIdx& x, int local, int rows, int K, int box) {
      ok = ok && make_tmap_3d(m, matp(c, blk(x, 0, local)), K, rows, d.N, blk_stride_bytes(c, x, local), box);
    };
    auto amap = [&](CUtensorMap* m, const void* p, int rows, int K, int box) {
      ok = ok && make_tmap_3d(m, p, K, rows, 1, 0, box);
    };
    // weight boxes: the tile's rows, or half of them for CTA pairs
    auto wbox = [](const GemmPlan& p) { return p.pair ? p.bn / 2 : p.bn; };
    const int bnv_qkv = wbox(c->p_v_qkv), bnv_o = wbox(c->p_v_o), bnv_f1 = wbox(c->p_v_f1), bnv_f2 = wbox(c->p_v_f2);
    const int bna = c->p_a_qkv.bn;
    amap(&c->m_hv, c->h_v, d.Mv, d.dv, 128);
    amap(&c->m_ov, c->o_v, d.Mv, d.A, 128);
    amap(&c->m_fv, c->f_v, d.Mv, d.Fv, 128);
    wmap(&c->m_w_qkv_v, c->ev, kQkvW, 3 * d.A, d.dv, bnv_qkv);
    wmap(&c->m_w_o_v, c->ev, kOW, d.dv, d.A, bnv_o);
    wmap(&c->m_w_f1_v, c->ev, kF1W, d.Fv, d.dv, bnv_f1);
    wmap(&c->m_w_f2_v, c->ev, kF2W, d.dv, d.Fv, bnv_f2);
    if (d.Pv > 0) {
      amap(&c->m_xvin, c->x_vin, d.Mv, d.Pv, 128);
      amap(&c->m_w_vin, matp(c, c->ev.inw), d.dv, d.Pv, c->p_v_in.bn);
    }
    if (cfg->video_has_output) amap(&c->m_w_vout, matp(c, c->ev.outw), d.Pv, d.dv, c->p_v_out.bn);
    amap(&c->m_w_in, matp(c, c->ea.inw), d.da, d.Kin, 128);
    wmap(&c->m_w_qkv_a, c->ea, kQkvW, 3 * d.A, d.da + d.r, 128);
    wmap(&c->m_w_o_a, c->ea, kOW, d.da, d.A + d.r, 128);
    wmap(&c->m_w_f1_a, c->ea, kF1W, d.Fa, d.da + d.r, 128);
    wmap(&c->m_w_f2_a, c->ea, kF2W, d.da, d.Fa + d.r, 128);
    if (d.r > 0) {
      wmap(&c->m_la_qkv, c->ea, kQkvLa, d.r, d.da, 128);
      wmap(&c->m_la_o, c->ea, kOLa, d.r, d.A, 128);
      wmap(&c->m_la_f1, c->ea, kF1La, d.r, d.da, 128);
      wmap(&c->m_la_f2, c->ea, kF2La, d.r, d.Fa, 128);
    }
    amap(&c->m_w_out, matp(c, c->ea.outw), d.Pa, d.da, 128);
    amap(&c->m_ain, c->a_in, d.Ma, d.Kin, bna);
    amap(&c->m_ha, c->h_a, d.Ma, d.lh, bna);
    amap(&c->m_oa, c->o_a, d.Ma, d.lo, bna);
    amap(&c->m_fa, c->f_a, d.Ma, d.lf, bna);
    ok = ok && make_tmap_3d(&c->m_qv, c->q_v, d.Dh, d.Lv, d.B * d.H, (size_t)d.Lv * d.Dh * 2, 128);
    ok = ok && make_tmap_3d(&c->m_cache, c->kv, d.Dh, d.Ltot, 2 * d.N * d.B * d.H, (size_t)d.Ltot * d.Dh * 2, 64);
    ok = ok && make_tmap_sw128(&c->m_xv_out, c->x_v, 4, d.dv, d.Mv, 1, 0, 32, 32);
    ok = ok && make_tmap_sw128(&c->m_fv_out, c->f_v, 2, d.Fv, d.Mv, 1, 0, 64, 32);
    ok = ok && make_tmap_sw128(&c->m_qv_out, c->q_v, 2, d.Dh, d.Lv, d.B * d.H, (size_t)d.Lv * d.Dh * 2, 64, 32);
    ok = ok && make_tmap_sw128(&c->m_cache_out, c->kv, 2, d.Dh, d.Ltot, 2 * d.N * d.B * d.H,
                               (size_t)d.Ltot * d.Dh * 2, 64, 32);
    if (!ok) return fail(c, WAM_ERR_CUDA, "tensor map creation failed");

    // Persistent action-block path (opt-in, WAM_ACTION_BLOCKS=1): bf16
    // without LoRA, at most 32 action tokens per chunk, action width a
    // multiple of 64 up to 768 (the block's B operand and one attention unit
    // share a 48 KB region).  Off by default: on the config-2 / config-3
    // chunks its launches (about 80 us per block, latency of the phase
    // chain) are slower than the per-operation kernels.
    const char* abv = getenv("WAM_ACTION_BLOCKS");
    const bool ab_want = abv && abv[0] == '1';
    if (ab_want && d.r == 0 && d.Ma <= 32 && d.da % 64 == 0 && d.da <= 768 && d.Fa % 64 == 0 && d.A % 64 == 0 &&
        d.Fa <= 4096 && d.A <= 4096) {
      int nsm = 148;
      CK(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, c->device));
      c->ab_ctas = nsm;
      int vctas_used = std::max(1, nsm * 73 / 100);
      if (const char* v = getenv("WAM_VIDEO_GEMM_CTAS")) {
        const int n = atoi(v);
        if (n > 0) vctas_used = std::min(n, nsm);
      }
      c->ab_ctas_overlap = std::max(8, nsm - vctas_used);
      if (const char* v = getenv("WAM_ACTION_BLOCK_CTAS")) {
        const int n = atoi(v);
        if (n > 0) c->ab_ctas_overlap = std::min(n, nsm);
      }
      c->ab_ks_in = action_block_ks(d.da, d.Kin, nsm);
      c->ab_ks_qkv = action_block_ks(3 * d.A, d.da, nsm);
      c->ab_ks_o = action_block_ks(d.da, d.A, nsm);
      c->ab_ks_f1 = action_block_ks(d.Fa, d.da, nsm);
      c->ab_ks_f2 = action_block_ks(d.da, d.Fa, nsm);
      c->ab_ks_out = action_block_ks(d.Pa, d.da, nsm);
      action_block_attn_plan(d.Lv + d.La, d.B * d.H, nsm, &c->ab_splits, &c->ab_keys);
      bool fits = (3 * d.A + 127) / 128 <= 64 && (d.Fa + 127) / 128 <= 64 && d.da % 128 == 0 && d.Dh == 64;
      for (int g : {c->ab_ctas, c->ab_ctas_overlap}) {
        fits = fits && action_block_fits(d.da, d.Kin, c->ab_ks_in, g) && action_block_fits(3 * d.A, d.da, c->ab_ks_qkv, g) &&
               action_block_fits(d.da, d.A, c->ab_ks_o, g) && action_block_fits(d.Fa, d.da, c->ab_ks_f1, g) &&
               action_block_fits(d.da, d.Fa, c->ab_ks_f2, g) && action_block_fits(d.Pa, d.da, c->ab_ks_out, g);
      }
      if (fits) {
        auto units = [&](int n_out, int ks) { return ((n_out + 127) / 128) * ks; };
        int mu = std::max({units(d.da, c->ab_ks_in), units(3 * d.A, c->ab_ks_qkv), units(d.da, c->ab_ks_o),
                           units(d.Fa, c->ab_ks_f1), units(d.da, c->ab_ks_f2), units(d.Pa, c->ab_ks_out)});
        CK(prepare_action_block());
        c->ab_ws_half = action_block_ws_floats(mu) / 2;
        RET(dalloc(c, &c->ab_ws, action_block_ws_floats(mu) * 4));
        RET(dalloc(c, &c->ab_ws_attn, action_block_attn_ws_floats(d.B, d.H, c->ab_splits) * 4));
        RET(dalloc(c, &c->ab_ss, (size_t)2 * (d.da / 128) * d.Ma * 4));
        RET(dalloc(c, &c->ab_cnt, (size_t)action_block_cnt_ints() * 4));
        RET(dalloc(c, &c->ab_cnt_attn, (size_t)d.B * d.H * 4));
        bool mok = make_tmap_3d(&c->m_qa128, c->q_a, d.Dh, d.La, d.B * d.H, (size_t)d.La * d.Dh * 2, 128) &&
                   make_tmap_3d(&c->m_cache_ab, c->kv, d.Dh, d.Ltot, 2 * d.N * d.B * d.H, (size_t)d.Ltot * d.Dh * 2,
                                c->ab_keys);
        if (!mok) return fail(c, WAM_ERR_CUDA, "tensor map creation failed");
        const CUtensorMap* mm[kActionBlockMaps] = {&c->m_w_qkv_a, &c->m_w_o_a, &c->m_w_f1_a, &c->m_w_f2_a,
                                                   &c->m_w_in,    &c->m_w_out, &c->m_oa,    &c->m_fa,
                                                   &c->m_ain,     &c->m_qa128, &c->m_cache_ab};
        for (int k = 0; k < kActionBlockMaps; ++k) c->ab_maps.m[k] = *mm[k];
        c->ab_on = true;
      }
    }
  }

  c->ev_kv.resize(d.N);
  c->ev_kv_cap.resize(d.N);
  c->ev_used.resize(d.N);
  for (int i = 0; i < d.N; ++i) {
    CK(cudaEventCreateWithFlags(&c->ev_kv[i], cudaEventDisableTiming));
    CK(cudaEventCreateWithFlags(&c->ev_kv_cap[i], cudaEventDisableTiming));
    CK(cudaEventCreateWithFlags(&c->ev_used[i], cudaEventDisableTiming));
  }
  for (auto* e : {&c->ev_fork, &c->ev_join, &c->ev_pre, &c->ev_post})
    CK(cudaEventCreateWithFlags(e, cudaEventDisableTiming));
  CK(cudaStreamCreateWithFlags(&c->cap_v, cudaStreamNonBlocking));
  CK(cudaStreamCreateWithFlags(&c->cap_a, cudaStreamNonBlocking));
  CK(cudaDeviceSynchronize());
  *out = holder.release();
  return WAM_OK;
}

wam_status wam_video_forward(wam_ctx* c, const float* video, const float* cond, float t_video, void* stream) {
  if (!c || !video || (c->d.Lc > 0 && !cond) || c->d.Pv > 0 || !(t_video >= 0.f && t_video <= 1.f))
    return fail(c, WAM_ERR_INVALID_ARG, "wam_video_forward: bad arguments");
  cudaStream_t s = (cudaStream_t)stream;
  VideoIo v{};
  v.video = video;
  v.cond = cond;
  v.t = t_video;
  CK(launch_set_video_io(c->vio_eager, v, s));
  RET(enqueue_video(c, s, c->vio_eager, false, c->ev_kv.data(), true));
  c->video_done = true;
  return WAM_OK;
}

wam_status wam_action_step(wam_ctx* c, float* actions, float t_from, float t_to, void* stream) {
  if (!c || !actions) return fail(c, WAM_ERR_INVALID_ARG, "wam_action_step: null argument");
  if (!(t_from > t_to && t_to >= 0.f && t_from <= 1.f))
    return fail(c, WAM_ERR_INVALID_ARG, "wam_action_step: need 1 >= t_from > t_to >= 0");
  if (!c->video_done) return fail(c, WAM_ERR_STATE, "wam_action_step before wam_video_forward");
  cudaStream_t s = (cudaStream_t)stream;
  const Dims& d = c->d;
  ActionIo a{};
  a.a_in = actions;
  a.a_out = actions;
  a.sched[0] = t_from;
  a.sched[1] = t_to;
  a.steps = 1;
  CK(launch_set_action_io(c->aio_eager, a, s));
  CK(launch_init_action(c->aio_eager, c->a_state, d.bf16 ? c->a_in : nullptr, d.bf16, d.Ma, d.Pa, d.Kin, s));
  RET(enqueue_action_step(c, s, c->aio_eager, 0, c->ev_kv.data(), true));
  CK(launch_copy_out(c->aio_eager, c->a_state, d.Ma * d.Pa, s));
  return WAM_OK;
}

wam_status wam_infer_chunk(wam_ctx* c, const float* video, const float* cond, const float* noise, float* out, int S,
                           const float* t_sched, int mode, int use_graph, void* stream_video, void* stream_action) {
  if (!c) return WAM_ERR_INVALID_ARG;
  if (!video || !noise || !out || (c->d.Lc > 0 && !cond) || c->d.Pv > 0)
    return fail(c, WAM_ERR_INVALID_ARG, "wam_infer_chunk: null buffer or patch-input model");
  if (S < 1 || S > kMaxSteps) return fail(c, WAM_ERR_INVALID_ARG, "wam_infer_chunk: S out of range");
  if (mode != WAM_SCHED_SEQUENTIAL && mode != WAM_SCHED_CEWP)
    return fail(c, WAM_ERR_INVALID_ARG, "wam_infer_chunk: bad mode");
  ActionIo a{};
  for (int j = 0; j <= S; ++j) a.sched[j] = t_sched ? t_sched[j] : (float)(S - j) / (float)S;
  if (!valid_schedule(a.sched, S)) return fail(c, WAM_ERR_INVALID_ARG, "wam_infer_chunk: schedule not decreasing in [0,1]");
  a.steps = S;
  a.a_in = noise;
  a.a_out = out;
  VideoIo v{};
  v.video = video;
  v.cond = cond;
  v.t = 0.f;
  cudaStream_t sv = (cudaStream_t)stream_video, sa = (cudaStream_t)stream_action;
  if (mode == WAM_SCHED_CEWP && sa == sv) return fail(c, WAM_ERR_INVALID_ARG, "CEWP needs two distinct streams");
  CK(cudaEventRecord(c->ev_pre, sa));
  CK(cudaStreamWaitEvent(sv, c->ev_pre, 0));
  RET(set_chunk_io(c, v, a, sv));
  return run_chunk(c, S, mode, use_graph, false, sv, sa);
}

wam_status wam_infer_chunk_host(wam_ctx* c, const float* hv, const float* hc, const float* hn, float* hout, int S,
                                const float* t_sched, int mode, int use_graph, void* stream_video, void* stream_action) {
  if (!c || !hv || !hn || !hout || (c->d.Lc > 0 && !hc)) return fail(c, WAM_ERR_INVALID_ARG, "null host buffer");
  const Dims& d = c->d;
  const size_t nv = (size_t)d.B * d.Lvid * d.dv, nc = (size_t)d.B * d.Lc * d.dv, nn = (size_t)d.Ma * d.Pa;
  // staging allocated on first use; each buffer on its own, so a failed
  // allocation is retried by the next call instead of leaving a gap
  if (!c->h_video) RET(dalloc(c, &c->h_video, nv * 4));
  if (!c->h_cond) RET(dalloc(c, &c->h_cond, nc * 4));
  if (!c->h_noise) RET(dalloc(c, &c->h_noise, nn * 4));
  if (!c->h_out) RET(dalloc(c, &c->h_out, nn * 4));
  cudaStream_t sv = (cudaStream_t)stream_video;
  CK(cudaMemcpyAsync(c->h_video, hv, nv * 4, cudaMemcpyHostToDevice, sv));
  if (nc) CK(cudaMemcpyAsync(c->h_cond, hc, nc * 4, cudaMemcpyHostToDevice, sv));
  CK(cudaMemcpyAsync(c->h_noise, hn, nn * 4, cudaMemcpyHostToDevice, sv));
  RET(wam_infer_chunk(c, c->h_video, nc ? c->h_cond : nullptr, c->h_noise, c->h_out, S, t_sched, mode, use_graph,
                      stream_video, stream_action));
  CK(cudaMemcpyAsync(hout, c->h_out, nn * 4, cudaMemcpyDeviceToHost, sv));
  CK(cudaStreamSynchronize(sv));
  return WAM_OK;
}

wam_status wam_joint_one_step(wam_ctx* c, const float* vclean, const float* veps, const float* aclean,
                              const float* aeps, float u_v, float u_a, float s_v, float s_a, float* vout, float* aout,
                              int mode, int use_graph, void* stream_video, void* stream_action) {
  if (!c) return WAM_ERR_INVALID_ARG;
  if (c->d.Pv <= 0 || !c->cfg.video_has_output)
    return fail(c, WAM_ERR_UNSUPPORTED, "wam_joint_one_step needs a patch-input model with a video output");
  if (!vclean || !veps || !aclean || !aeps || !vout || !aout || !(u_v >= 0.f && u_v <= 1.f) ||
      !(u_a > 0.f && u_a <= 1.f) || !(s_v > 0.f) || !(s_a > 0.f))
    return fail(c, WAM_ERR_INVALID_ARG, "wam_joint_one_step: bad arguments");
  cudaStream_t sv = (cudaStream_t)stream_video, sa = (cudaStream_t)stream_action;
  if (mode == WAM_SCHED_CEWP && sa == sv) return fail(c, WAM_ERR_INVALID_ARG, "CEWP needs two distinct streams");
  VideoIo v{};
  v.video = vclean;
  v.eps = veps;
  v.video_out = vout;
  v.u = u_v;
  v.shift = s_v;
  ActionIo a{};
  a.a_in = aeps;
  a.a_clean = aclean;
  a.a_out = aout;
  a.u = u_a;
  a.shift = s_a;
  a.steps = 1;
  CK(cudaEventRecord(c->ev_pre, sa));
  CK(cudaStreamWaitEvent(sv, c->ev_pre, 0));
  RET(set_chunk_io(c, v, a, sv));
  return run_chunk(c, 1, mode, use_graph, true, sv, sa);
}

namespace {
// S eager Euler steps of the action expert of `c` along sched[0..S] from
// dev_in into dev_out, on `s`, with the block K/V already in c's cache.
wam_status run_action_steps(wam_ctx* c, cudaStream_t s, const float* dev_in, float* dev_out, const float* sched,
                            int S) {
  const Dims& d = c->d;
  ActionIo a{};
  a.a_in = dev_in;
  a.a_out = dev_out;
  for (int j = 0; j <= S; ++j) a.sched[j] = sched[j];
  a.steps = S;
  CK(launch_set_action_io(c->aio_tacd, a, s));
  CK(launch_init_action(c->aio_tacd, c->a_state, d.bf16 ? c->a_in : nullptr, d.bf16, d.Ma, d.Pa, d.Kin, s));
  if (!c->kv_flag_clean) RET(clear_kv_flag(c, s));  // an earlier sequence stopped before its end
  for (int j = 0; j < S; ++j) RET(enqueue_action_step(c, s, c->aio_tacd, j, nullptr, false));
  CK(launch_copy_out(c->aio_tacd, c->a_state, d.Ma * d.Pa, s));
  if (S > 1) RET(clear_kv_flag(c, s));
  return WAM_OK;
}
}  // namespace

wam_status wam_tacd_targets(wam_ctx* c, wam_ctx* ema, const float* video, const float* cond, const float* a_clean,
                            const float* eps, float t, int K, float lambda, float* u_ta, float* v_student,
                            float* u_cd, float* losses, float* a_t_out, float* a0_teacher_out, void* stream) {
  if (!c || !ema) return WAM_ERR_INVALID_ARG;
  const Dims& d = c->d;
  if (!video || !a_clean || !eps || !losses || (d.Lc > 0 && !cond) || d.Pv > 0 || !(t > 0.f && t <= 1.f) || K < 1 ||
      K > kMaxSteps)
    return fail(c, WAM_ERR_INVALID_ARG, "wam_tacd_targets: bad arguments");
  if (d.r <= 0 || memcmp(&c->cfg, &ema->cfg, sizeof c->cfg) != 0 || c->device != ema->device)
    return fail(c, WAM_ERR_INVALID_ARG, "wam_tacd_targets: student and EMA need the same LoRA model on one device");
  cudaStream_t s = (cudaStream_t)stream;
  const size_t n = (size_t)d.Ma * d.Pa;
  for (float** p : {&c->td_at, &c->td_as, &c->td_a0, &c->td_fs, &c->td_fe})
    if (!*p) RET(dalloc(c, p, n * 4));
  if (!c->aio_tacd) RET(dalloc(c, &c->aio_tacd, sizeof(ActionIo)));
  if (ema != c && !ema->aio_tacd) RET(dalloc(ema, &ema->aio_tacd, sizeof(ActionIo)));
  // teacher grid t_k = t k / K (k = K .. 0); s = t (K - 1) / K is its first point
  float grid[kMaxSteps + 1];
  for (int k = 0; k <= K; ++k) grid[k] = (float)((double)t * (double)(K - k) / (double)K);
  const float s_pt = grid[1];
  // a_t, and the frozen video expert once (t_v = 0) into the student's cache
  CK(launch_tacd_noise(a_clean, eps, t, c->td_at, (int)n, s));
  VideoIo v{};
  v.video = video;
  v.cond = cond;
  CK(launch_set_video_io(c->vio_eager, v, s));
  RET(enqueue_video(c, s, c->vio_eager, false, nullptr, false));
  // teacher: the base weights (LoRA scale 0 adds exact zeros), K Euler steps
  // from (a_t, t) to 0; the first state is a~_s
  const float scale = c->cfg.lora_scale;
  c->cfg.lora_scale = 0.f;
  wam_status st = run_action_steps(c, s, c->td_at, c->td_as, grid, 1);
  if (st == WAM_OK) st = K > 1 ? run_action_steps(c, s, c->td_as, c->td_a0, grid + 1, K - 1) : WAM_OK;
  c->cfg.lora_scale = scale;
  RET(st);
  const float* a0T = K > 1 ? c->td_a0 : c->td_as;
  // student endpoint f(a_t, t) = a_t - t v (one step t -> 0)
  const float sched_st[2] = {t, 0.f};
  RET(run_action_steps(c, s, c->td_at, c->td_fs, sched_st, 1));
  // EMA endpoint f^-(a~_s, s) over the same K/V (s = 0: the endpoint map is the identity)
  const float* fe = c->td_as;
  if (s_pt > 0.f) {
    if (ema != c) {
      const size_t kv_bytes = (size_t)2 * d.N * d.B * d.H * d.Ltot * d.Dh * c->esz;
      CK(cudaMemcpyAsync(ema->kv, c->kv, kv_bytes, cudaMemcpyDeviceToDevice, s));
    }
    const float sched_ema[2] = {s_pt, 0.f};
    RET(run_action_steps(ema, s, c->td_as, c->td_fe, sched_ema, 1));
    fe = c->td_fe;
  }
  if (a_t_out) CK(cudaMemcpyAsync(a_t_out, c->td_at, n * 4, cudaMemcpyDeviceToDevice, s));
  if (a0_teacher_out) CK(cudaMemcpyAsync(a0_teacher_out, a0T, n * 4, cudaMemcpyDeviceToDevice, s));
  CK(launch_tacd_targets(c->td_at, a0T, c->td_fs, fe, t, lambda, d.B, d.La * d.Pa, u_ta, v_student, u_cd, losses, s));
  return WAM_OK;
}

wam_status wam_infer_chunk_multistep(wam_ctx* c, const float* video_eps, const float* noise, float* video_out,
                                     float* actions_out, int n_video, const float* sched_v, int S,
                                     const float* t_sched, int mode, int use_graph, void* stream_video,
                                     void* stream_action) {
  if (!c) return WAM_ERR_INVALID_ARG;
  if (c->d.Pv <= 0 || !c->cfg.video_has_output)
    return fail(c, WAM_ERR_UNSUPPORTED, "wam_infer_chunk_multistep needs a patch-input model with a video output");
  if (!video_eps || !noise || !video_out || !actions_out || n_video < 1 || n_video > kMaxSteps || S < 1 ||
      S > kMaxSteps || (mode != WAM_SCHED_SEQUENTIAL && mode != WAM_SCHED_CEWP))
    return fail(c, WAM_ERR_INVALID_ARG, "wam_infer_chunk_multistep: bad arguments");
  cudaStream_t sv = (cudaStream_t)stream_video, sa = (cudaStream_t)stream_action;
  if (mode == WAM_SCHED_CEWP && sa == sv) return fail(c, WAM_ERR_INVALID_ARG, "CEWP needs two distinct streams");
  VideoIo v{};
  for (int j = 0; j <= n_video; ++j) v.vsched[j] = sched_v ? sched_v[j] : (float)(n_video - j) / (float)n_video;
  if (!valid_schedule(v.vsched, n_video) || v.vsched[0] != 1.f)
    return fail(c, WAM_ERR_INVALID_ARG, "wam_infer_chunk_multistep: video schedule must fall from 1 within [0,1]");
  v.vsteps = n_video;
  v.video = video_eps;  // the latents at level 1 are the noise itself: (1 - 1) x + 1 eps
  v.eps = video_eps;
  v.t = 1.f;
  v.video_out = video_out;
  ActionIo a{};
  for (int j = 0; j <= S; ++j) a.sched[j] = t_sched ? t_sched[j] : (float)(S - j) / (float)S;
  if (!valid_schedule(a.sched, S)) return fail(c, WAM_ERR_INVALID_ARG, "wam_infer_chunk_multistep: bad schedule");
  a.steps = S;
  a.a_in = noise;
  a.a_out = actions_out;
  CK(cudaEventRecord(c->ev_pre, sa));
  CK(cudaStreamWaitEvent(sv, c->ev_pre, 0));
  RET(set_chunk_io(c, v, a, sv));
  return run_chunk(c, S, mode, use_graph, false, sv, sa, n_video);
}

wam_status wam_profile_chunk(wam_ctx* c, const float* video, const float* cond, const float* noise, float* out, int S,
                             void* stream, float* host_ms, int* host_counts) {
  if (!c || !host_ms || !host_counts) return WAM_ERR_INVALID_ARG;
  if (!video || !noise || !out || (c->d.Lc > 0 && !cond) || c->d.Pv > 0 || S < 1 || S > kMaxSteps)
    return fail(c, WAM_ERR_INVALID_ARG, "wam_profile_chunk: bad arguments");
  cudaStream_t s = (cudaStream_t)stream;
  ActionIo a{};
  for (int j = 0; j <= S; ++j) a.sched[j] = (float)(S - j) / (float)S;
  a.steps = S;
  a.a_in = noise;
  a.a_out = out;
  VideoIo v{};
  v.video = video;
  v.cond = cond;
  RET(set_chunk_io(c, v, a, s));
  // Capture the sequential chunk with an event-record node around every
  // launch, then replay it: the kernels run back to back as in the timed
  // graph, without host launch latency between them.
  CK(cudaStreamSynchronize(s));
  c->prof.clear();
  c->prof_next = 0;
  c->prof_on = true;
  c->launches = 0;
  cudaGraph_t graph = nullptr;
  CK(cudaStreamBeginCapture(c->cap_v, cudaStreamCaptureModeThreadLocal));
  wam_status st = enqueue_chunk(c, S, WAM_SCHED_SEQUENTIAL, false, c->cap_v, c->cap_v, c->ev_kv_cap.data());
  c->prof_on = false;
  cudaError_t ce = cudaStreamEndCapture(c->cap_v, &graph);
  if (st != WAM_OK) {
    if (graph) cudaGraphDestroy(graph);
    return st;
  }
  CK(ce);
  cudaGraphExec_t exec = nullptr;
  ce = cudaGraphInstantiate(&exec, graph, 0);
  cudaGraphDestroy(graph);
  CK(ce);
  ce = cudaGraphLaunch(exec, s);
  if (ce == cudaSuccess) ce = cudaStreamSynchronize(s);
  cudaGraphExecDestroy(exec);
  CK(ce);
  for (int k = 0; k < WAM_PROF_CLASSES; ++k) {
    host_ms[k] = 0.f;
    host_counts[k] = 0;
  }
  for (auto& r : c->prof) {
    float ms = 0.f;
    CK(cudaEventElapsedTime(&ms, r.a, r.b));
    host_ms[r.cls] += ms;
    host_counts[r.cls] += 1;
  }
  return WAM_OK;
}

wam_status wam_trace_chunk(wam_ctx* c, const float* video, const float* cond, const float* noise, float* out, int S,
                           int mode, void* stream_video, void* stream_action, float* host_ms, int capacity,
                           int* count) {
  if (!c || !host_ms || !count || capacity < 0) return WAM_ERR_INVALID_ARG;
  if (!video || !noise || !out || (c->d.Lc > 0 && !cond) || c->d.Pv > 0 || S < 1 || S > kMaxSteps ||
      (mode != WAM_SCHED_SEQUENTIAL && mode != WAM_SCHED_CEWP))
    return fail(c, WAM_ERR_INVALID_ARG, "wam_trace_chunk: bad arguments");
  cudaStream_t sv = (cudaStream_t)stream_video, sa = (cudaStream_t)stream_action;
  if (mode == WAM_SCHED_CEWP && sa == sv) return fail(c, WAM_ERR_INVALID_ARG, "CEWP needs two distinct streams");
  ActionIo a{};
  for (int j = 0; j <= S; ++j) a.sched[j] = (float)(S - j) / (float)S;
  a.steps = S;
  a.a_in = noise;
  a.a_out = out;
  VideoIo v{};
  v.video = video;
  v.cond = cond;
  CK(cudaEventRecord(c->ev_pre, sa));
  CK(cudaStreamWaitEvent(sv, c->ev_pre, 0));
  RET(set_chunk_io(c, v, a, sv));
  CK(cudaStreamSynchronize(sv));
  // capture the chunk with timing events at the block boundaries, replay once
  c->trace.clear();
  c->trace_on = true;
  cudaGraph_t graph = nullptr;
  CK(cudaStreamBeginCapture(c->cap_v, cudaStreamCaptureModeThreadLocal));
  trace_mark(c, c->cap_v, WAM_TRACE_START, 0);
  wam_status st = enqueue_chunk(c, S, mode, false, c->cap_v, mode == WAM_SCHED_CEWP ? c->cap_a : c->cap_v,
                                c->ev_kv_cap.data());
  if (st == WAM_OK) trace_mark(c, c->cap_v, WAM_TRACE_END, 0);
  c->trace_on = false;
  cudaError_t ce = cudaStreamEndCapture(c->cap_v, &graph);
  if (st != WAM_OK) {
    if (graph) cudaGraphDestroy(graph);
    return st;
  }
  CK(ce);
  cudaGraphExec_t exec = nullptr;
  ce = cudaGraphInstantiate(&exec, graph, 0);
  cudaGraphDestroy(graph);
  CK(ce);
  // one warm replay, then the timed one
  for (int r = 0; r < 2 && ce == cudaSuccess; ++r) {
    ce = cudaGraphLaunch(exec, sv);
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(sv);
  }
  cudaGraphExecDestroy(exec);
  CK(ce);
  // records: (kind, block, step, ms since the start mark)
  *count = (int)c->trace.size();
  for (size_t k = 0; k < c->trace.size() && (int)k < capacity; ++k) {
    float ms = 0.f;
    CK(cudaEventElapsedTime(&ms, c->trace[0].e, c->trace[k].e));
    host_ms[4 * k + 0] = (float)c->trace[k].kind;
    host_ms[4 * k + 1] = (float)c->trace[k].block;
    host_ms[4 * k + 2] = (float)c->trace[k].step;
    host_ms[4 * k + 3] = ms;
  }
  return WAM_OK;
}

wam_status wam_export_params(wam_ctx* c, float* host, size_t* nbytes) {
  if (!c || !nbytes) return WAM_ERR_INVALID_ARG;
  size_t total = 0;
  for (auto& e : c->params) total += e.count();
  if (!host) {
    *nbytes = total * 4;
    return WAM_OK;
  }
  if (*nbytes < total * 4) return fail(c, WAM_ERR_INVALID_ARG, "export buffer too small");
  float* tmp = nullptr;
  size_t mx = 0;
  for (auto& e : c->params) mx = std::max(mx, e.count());
  RET(dalloc(c, &tmp, mx * 4));
  size_t at = 0;
  wam_status st = WAM_OK;
  for (size_t p = 0; p < c->params.size() && st == WAM_OK; ++p) {
    const PEntry& e = c->params[p];
    const void* src = e.matrix ? matp(c, (int)p) : (const void*)vecp(c, (int)p);
    cudaError_t ce = launch_to_f32(src, e.matrix && c->d.bf16, tmp, e.count(), e.cols, e.matrix ? e.ld : e.cols, 0);
    if (ce == cudaSuccess) ce = cudaMemcpy(host + at, tmp, e.count() * 4, cudaMemcpyDeviceToHost);
    if (ce != cudaSuccess) st = fail(c, WAM_ERR_CUDA, "export: %s", cudaGetErrorString(ce));
    at += e.count();
  }
  cudaFree(tmp);
  c->mem_used -= mx * 4;
  *nbytes = total * 4;
  return st;
}

wam_status wam_import_params(wam_ctx* c, const float* host, size_t nbytes) {
  if (!c || !host) return WAM_ERR_INVALID_ARG;
  size_t total = 0;
  for (auto& e : c->params) total += e.count();
  if (nbytes != total * 4) return fail(c, WAM_ERR_INVALID_ARG, "import size mismatch");
  CK(cudaDeviceSynchronize());
  std::vector<uint16_t> hb;
  size_t at = 0;
  for (size_t p = 0; p < c->params.size(); ++p) {
    const PEntry& e = c->params[p];
    const float* src = host + at;
    at += e.count();
    if (!e.matrix) {
      std::vector<float> v(src, src + e.count());
      if (c->d.bf16)
        for (auto& f : v) {
          uint32_t b;
          memcpy(&b, &f, 4);
          b = (b + 0x7FFFu + ((b >> 16) & 1u)) & 0xFFFF0000u;
          memcpy(&f, &b, 4);
        }
      CK(cudaMemcpy(vecp(c, (int)p), v.data(), e.count() * 4, cudaMemcpyHostToDevice));
      continue;
    }
    // rows of `cols` values into rows of pitch ld (other columns of the rows,
    // e.g. the LoRA B factor inside a weight matrix, are left alone)
    if (c->d.bf16) {
      hb.assign((size_t)e.rows * e.cols, 0);
      for (size_t i = 0; i < hb.size(); ++i) {
        uint32_t b;
        memcpy(&b, &src[i], 4);
        hb[i] = (uint16_t)((b + 0x7FFFu + ((b >> 16) & 1u)) >> 16);
      }
      CK(cudaMemcpy2D(matp(c, (int)p), (size_t)e.ld * 2, hb.data(), (size_t)e.cols * 2, (size_t)e.cols * 2, e.rows,
                      cudaMemcpyHostToDevice));
    } else {
      CK(cudaMemcpy2D(matp(c, (int)p), (size_t)e.ld * 4, src, (size_t)e.cols * 4, (size_t)e.cols * 4, e.rows,
                      cudaMemcpyHostToDevice));
    }
  }
  return WAM_OK;
}

wam_status wam_read_kv(wam_ctx* c, int block, int which, float* host, size_t* nbytes) {
  if (!c || !nbytes || block < 0 || block >= c->d.N || (which != 0 && which != 1)) return WAM_ERR_INVALID_ARG;
  const Dims& d = c->d;
  const size_t n = (size_t)d.B * d.H * d.Ltot * d.Dh;
  if (!host) {
    *nbytes = n * 4;
    return WAM_OK;
  }
  if (*nbytes < n * 4) return fail(c, WAM_ERR_INVALID_ARG, "read_kv buffer too small");
  CK(cudaDeviceSynchronize());
  float* tmp = nullptr;
  RET(dalloc(c, &tmp, n * 4));
  cudaError_t ce = launch_to_f32(which ? vcache(c, block) : kcache(c, block), d.bf16, tmp, n, 1, 1, 0);
  if (ce == cudaSuccess) ce = cudaMemcpy(host, tmp, n * 4, cudaMemcpyDeviceToHost);
  cudaFree(tmp);
  c->mem_used -= n * 4;
  CK(ce);
  return WAM_OK;
}

wam_status wam_check_device_status(wam_ctx* c) {
  if (!c) return WAM_ERR_INVALID_ARG;
  CK(cudaDeviceSynchronize());
  unsigned st = 0;
  CK(cudaMemcpy(&st, c->status, 4, cudaMemcpyDeviceToHost));
  if (st) {
    // A kernel that gave up may have left its tickets, counters or grid
    // barrier mid-way: clear them so that the next call starts clean.
    CK(cudaMemset(c->status, 0, 4));
    if (c->tk_gemm) CK(cudaMemset(c->tk_gemm, 0, c->tk_gemm_bytes));
    if (c->tk_gemm_v) CK(cudaMemset(c->tk_gemm_v, 0, c->tk_gemm_v_bytes));
    if (c->na_cnt) CK(cudaMemset(c->na_cnt, 0, 3 * 4));
    if (c->ab_cnt) CK(cudaMemset(c->ab_cnt, 0, (size_t)action_block_cnt_ints() * 4));
    if (c->ab_cnt_attn) CK(cudaMemset(c->ab_cnt_attn, 0, (size_t)c->d.B * c->d.H * 4));
    if (c->tk_attn) CK(cudaMemset(c->tk_attn, 0, (size_t)c->d.B * c->d.H * 4));
    CK(cudaDeviceSynchronize());
    return fail(c, WAM_ERR_TIMEOUT, "device bounded wait gave up (status bits 0x%x)", st);
  }
  return WAM_OK;
}

wam_status wam_patchify(const float* frames, float* patches, int B, int F, int C, int H, int W, int p, int inverse,
                        void* stream) {
  if (!frames || !patches || B < 1 || F < 1 || C < 1 || p < 1 || H < p || W < p || H % p || W % p)
    return WAM_ERR_INVALID_ARG;
  return launch_patchify(inverse ? patches : frames, inverse ? const_cast<float*>(frames) : patches, B, F, C, H, W,
                         p, inverse != 0, (cudaStream_t)stream) == cudaSuccess
             ? WAM_OK
             : WAM_ERR_CUDA;
}

wam_status wam_test_peer_wait(int extra, unsigned long long limit_ns) {
  if (extra < 0 || (extra > 0 && limit_ns == 0)) return WAM_ERR_INVALID_ARG;
  if (extra == 0) limit_ns = 2000000000ull;  // the kernels' normal limit (2 s)
  return set_peer_wait_test(extra, limit_ns) == cudaSuccess ? WAM_OK : WAM_ERR_CUDA;
}

int wam_chunk_kernel_count(wam_ctx* c, int S) {
  if (!c) return -1;
  for (auto& kv : c->launch_counts)
    if ((kv.first >> 24) == S) return kv.second;
  return -1;
}

// ------------------------------------------------- single-op entry points --
namespace {
// One GEMM with bias into fp32 out[M, N] through the tcgen05 kernel (private
// workspace grown on demand).  Normal orientation: bn 128 or 256, `ctas`
// persistent CTAs (0: all SMs), pair = CTA pairs; swapped: `ctas` = CTAs per
// output tile.
wam_status op_linear_bf16(const void* x, const void* w, const float* bias, float* out, int M, int N, int K, bool swap,
                          int ctas, int bn_normal, bool pair, cudaStream_t s, bool csplit = false, bool cred = false) {
  if (K % 64) return WAM_ERR_INVALID_ARG;
  const int bn = swap ? (M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256) : bn_normal;
  if (swap && M > 256) return WAM_ERR_INVALID_ARG;
  if (!swap && (N % 32 || (bn != 128 && bn != 192 && bn != 256) || (pair && bn != 256))) return WAM_ERR_INVALID_ARG;
  static thread_local unsigned* status = nullptr;
  if (!status) {
    if (prepare_tc_gemm() != cudaSuccess) return WAM_ERR_CUDA;
    if (cudaMalloc(&status, 4) != cudaSuccess) return WAM_ERR_OOM;
    cudaMemset(status, 0, 4);
  }
  EpiArgs e;
  e.kind = kEpiStoreF32;
  e.bias = bias;
  e.out_f32 = out;
  e.ld_out = N;
  TcGemm g{};
  g.rows_a = swap ? N : M;
  g.rows_b = swap ? M : N;
  g.K = K;
  g.z_a = g.z_b = 0;
  g.bn = bn;
  g.splits = swap ? std::max(1, ctas) : 1;
  g.swap = swap;
  g.max_ctas = swap ? 0 : std::max(0, ctas);
  g.pair = pair;
  g.csplit = csplit;
  g.cred = swap && cred ? g.splits : 0;
  const size_t tickets = tc_gemm_tickets(g);
  static thread_local float* ws = nullptr;
  static thread_local int* tk = nullptr;
  static thread_local size_t ws_cap = 0, tk_cap = 0;
  const size_t need = tc_gemm_ws_floats(g);
  if (need > ws_cap) {
    if (ws) cudaFree(ws);
    ws = nullptr;
    ws_cap = 0;
    if (cudaMalloc(&ws, need * 4) != cudaSuccess) return WAM_ERR_OOM;
    ws_cap = need;
  }
  if (tickets > tk_cap) {
    if (tk) cudaFree(tk);
    tk = nullptr;
    tk_cap = 0;
    if (cudaMalloc(&tk, tickets * 4) != cudaSuccess) return WAM_ERR_OOM;
    if (cudaMemset(tk, 0, tickets * 4) != cudaSuccess) return WAM_ERR_CUDA;
    tk_cap = tickets;
  }
  CUtensorMap mx, mw, mo;
  const int wbox = swap ? 128 : (pair ? bn / 2 : bn);
  if (!make_tmap_3d(&mx, x, K, M, 1, 0, swap ? bn : 128) || !make_tmap_3d(&mw, w, K, N, 1, 0, wbox))
    return WAM_ERR_INVALID_ARG;
  if (!swap) {
    if (!make_tmap_sw128(&mo, out, 4, N, M, 1, 0, 32, 32)) return WAM_ERR_INVALID_ARG;
    e.map_o = &mo;
  }
  g.map_a = swap ? &mw : &mx;
  g.map_b = swap ? &mx : &mw;
  g.ws = ws;
  g.tickets = tk;
  g.status = status;
  return launch_tc_gemm(g, e, s) == cudaSuccess ? WAM_OK : WAM_ERR_CUDA;
}
}  // namespace

wam_status wam_op_linear(int dtype, const void* x, const void* w, const float* bias, float* out, int M, int N, int K,
                         int swap, int splits, void* stream) {
  if (!x || !w || !bias || !out || M < 1 || N < 1 || K < 1) return WAM_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (dtype == WAM_FP32) {
    EpiArgs e;
    e.kind = kEpiStoreF32;
    e.bias = bias;
    e.out_f32 = out;
    e.ld_out = N;
    return launch_f32_gemm((const float*)x, K, (const float*)w, M, N, K, e, s) == cudaSuccess ? WAM_OK : WAM_ERR_CUDA;
  }
  if (dtype != WAM_BF16) return WAM_ERR_INVALID_ARG;
  return op_linear_bf16(x, w, bias, out, M, N, K, swap != 0, splits, 128, false, s);
}

wam_status wam_op_linear_tiled(const void* x, const void* w, const float* bias, float* out, int M, int N, int K, int bn,
                               int mode, int ctas, void* stream) {
  if (!x || !w || !bias || !out || M < 1 || N < 1 || K < 1 || ctas < 0 || mode < 0 || mode > 3)
    return WAM_ERR_INVALID_ARG;
  if (mode == 2 && ctas % 2) return WAM_ERR_INVALID_ARG;  // clusters of two: an even grid
  if (mode == 3) {  // swapped, clusters of `ctas` CTAs per tile
    if (M > 64 || ctas < 2 || ctas > 8 || (K / 64) % ctas || (M <= 32 ? 32 : 64) % (4 * ctas))
      return WAM_ERR_INVALID_ARG;
    return op_linear_bf16(x, w, bias, out, M, N, K, true, ctas, 128, false, (cudaStream_t)stream, false, true);
  }
  return op_linear_bf16(x, w, bias, out, M, N, K, false, ctas, bn, mode == 1, (cudaStream_t)stream, mode == 2);
}

wam_status wam_op_attention_joint(const void* q, const void* k, const void* v, void* out, int B, int H, int Lq, int Lk,
                                  int Lcache, int ready, int splits, void* stream) {
  if (!q || !k || !v || !out || B < 1 || H < 1 || Lq < 1 || Lq > 64 || Lk < 1 || Lk > Lcache || ready < 0 ||
      ready > Lcache || splits < 0)
    return WAM_ERR_INVALID_ARG;
  static thread_local unsigned* status = nullptr;
  if (!status) {
    if (prepare_attention_joint() != cudaSuccess) return WAM_ERR_CUDA;
    if (cudaMalloc(&status, 4) != cudaSuccess) return WAM_ERR_OOM;
    if (cudaMemset(status, 0, 4) != cudaSuccess) return WAM_ERR_CUDA;
  }
  if (splits == 0) {
    int dev = 0, nsm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    splits = attention_joint_splits(B * H, Lq, Lk, nsm);
  }
  CUtensorMap mk, mv;
  const size_t mat = (size_t)Lcache * 64 * 2;
  if (!make_tmap_3d(&mk, k, 64, Lcache, B * H, mat, 64) || !make_tmap_3d(&mv, v, 64, Lcache, B * H, mat, 64))
    return WAM_ERR_INVALID_ARG;
  AttnJoint t;
  t.map_k = &mk;
  t.map_v = &mv;
  t.zk0 = t.zv0 = 0;
  t.q = q;
  t.out = out;
  t.B = B;
  t.H = H;
  t.Lq = Lq;
  t.Lk = Lk;
  t.ld_out = 0;
  t.ready = ready;
  t.splits = splits;
  t.status = status;
  return launch_attention_joint(t, (cudaStream_t)stream) == cudaSuccess ? WAM_OK : WAM_ERR_INVALID_ARG;
}

wam_status wam_op_norm_mod(int dtype, const float* x, void* h, int M, int d, const float* scale, const float* shift,
                           const float* gain, void* stream) {
  if (!x || !h || M < 1 || d < 4 || d % 4 || d > 1536 || (!gain && !scale) ||
      (dtype != WAM_BF16 && dtype != WAM_FP32))
    return WAM_ERR_INVALID_ARG;
  return launch_norm_mod(x, h, dtype == WAM_BF16, M, d, scale, shift, gain, (cudaStream_t)stream) == cudaSuccess
             ? WAM_OK
             : WAM_ERR_CUDA;
}

wam_status wam_op_attention(int dtype, const void* q, const void* k, const void* v, void* out, int B, int H, int Dh,
                            int Lq, int Lk, int Lcache, int splits, void* stream) {
  if (!q || !k || !v || !out || B < 1 || H < 1 || Lq < 1 || Lk < 1 || Lk > Lcache) return WAM_ERR_INVALID_ARG;
  AttnArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.out = out;
  a.B = B;
  a.H = H;
  a.Dh = Dh;
  a.Lq = Lq;
  a.Lk = Lk;
  a.Lcache = Lcache;
  a.splits = splits < 1 ? 1 : splits;
  a.ws = nullptr;
  a.tickets = nullptr;
  cudaStream_t s = (cudaStream_t)stream;
  if (dtype == WAM_FP32) return launch_attention_f32(a, s) == cudaSuccess ? WAM_OK : WAM_ERR_CUDA;
  if (dtype != WAM_BF16 || Dh != 64) return WAM_ERR_INVALID_ARG;
  if (a.splits == 1) {  // single pass: the tcgen05 kernel
    static thread_local unsigned* st = nullptr;
    if (!st) {
      if (prepare_attention_tc() != cudaSuccess) return WAM_ERR_CUDA;
      if (cudaMalloc(&st, 4) != cudaSuccess) return WAM_ERR_OOM;
      if (cudaMemset(st, 0, 4) != cudaSuccess) return WAM_ERR_CUDA;
    }
    CUtensorMap mq, mk, mv;
    if (!make_tmap_3d(&mq, q, 64, Lq, B * H, (size_t)Lq * 128, 128) ||
        !make_tmap_3d(&mk, k, 64, Lcache, B * H, (size_t)Lcache * 128, 64) ||
        !make_tmap_3d(&mv, v, 64, Lcache, B * H, (size_t)Lcache * 128, 64))
      return WAM_ERR_INVALID_ARG;
    AttnTc t;
    t.map_q = &mq;
    t.map_k = &mk;
    t.map_v = &mv;
    t.zq0 = t.zk0 = t.zv0 = 0;
    t.B = B;
    t.H = H;
    t.Lq = Lq;
    t.Lk = Lk;
    t.out = out;
    t.status = st;
    return launch_attention_tc(t, s) == cudaSuccess ? WAM_OK : WAM_ERR_CUDA;
  }
  if (a.splits > 1) {
    if (Lq > 64) return WAM_ERR_INVALID_ARG;
    static thread_local bool prepared = false;
    if (!prepared) {
      if (prepare_attention_bf16() != cudaSuccess) return WAM_ERR_CUDA;
      prepared = true;
    }
    static thread_local float* ws = nullptr;
    static thread_local int* tk = nullptr;
    static thread_local size_t cap = 0, tcap = 0;
    const size_t need = attention_ws_floats(B, H, Dh, Lq, a.splits);
    if (need > cap) {
      if (ws) cudaFree(ws);
      if (cudaMalloc(&ws, need * 4) != cudaSuccess) return WAM_ERR_OOM;
      cap = need;
    }
    if ((size_t)B * H > tcap) {
      if (tk) cudaFree(tk);
      if (cudaMalloc(&tk, (size_t)B * H * 4) != cudaSuccess) return WAM_ERR_OOM;
      if (cudaMemset(tk, 0, (size_t)B * H * 4) != cudaSuccess) return WAM_ERR_CUDA;
      tcap = (size_t)B * H;
    }
    a.ws = ws;
    a.tickets = tk;
  }
  return launch_attention_bf16(a, s) == cudaSuccess ? WAM_OK : WAM_ERR_CUDA;
}

}  // extern "C"
