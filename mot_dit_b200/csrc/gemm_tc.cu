// tcgen05 GEMM for sm_100a with the MoT block epilogues fused in.
//
// C[m, n] = sum_k X[m, k] W[n, k]: X = activations (tokens x K), W = a weight
// stored [out, in] (K contiguous).  Both operands are K-major bf16 tiles moved
// by TMA (128-byte swizzle) into a multi-stage shared-memory ring; one thread
// issues tcgen05.mma (M = 128, N = BN, K = 16) into an fp32 accumulator in
// tensor memory; four epilogue warps read it back with tcgen05.ld and apply
// the fused epilogue (bias, gate-residual, GELU, QK-norm + RoPE + K/V publish,
// Euler update, video endpoint).
//
// Schedule (stream-K): the k-blocks of all output tiles, tile after tile, form
// one range of W = tiles x KB blocks, and persistent CTA c of G owns blocks
// [W c / G, W (c+1) / G).  Every CTA gets the same amount of MMA work however
// the tile count falls on the SMs.  A tile whose k-range is shared by several
// CTAs is finished by the last of its pieces to arrive (integer ticket), which
// sums the fp32 partials in piece (= k) order: the result does not depend on
// timing.  The accumulator is double-buffered in TMEM (2 x BN columns): the
// MMA warp fills one while the epilogue warps drain the other.
//
// Split tiles.  Each piece takes an arrival ticket when its accumulator is
// ready.  Every piece but the last to arrive publishes its fp32 partial to the
// workspace and counts itself published; the last one waits (bounded) for
// those counts -- of pieces that have already arrived, so the wait never
// depends on a CTA that is not running -- and adds the partials, in piece
// order, to its own accumulator read from TMEM.  The last arrival is almost
// always piece 0, the final segment of its CTA: the shared-memory ring is
// idle by then, and the partials come in with bulk copies.
//
// Orientation.  Normal: A = X (128 tokens on TMEM lanes), B = W (BN features).
// Swapped (few tokens, e.g. the action expert's 32): A = W (128 features on
// TMEM lanes), B = X (BN tokens) -- the weight stream fills the 128-row MMA
// operand instead of padding the token dimension.
//
// Epilogue stores of the normal orientation go through shared memory: each
// epilogue warp writes its 32-row output box in the 128-byte-swizzled layout
// and one lane issues a TMA bulk-tensor store.  The gate-residual rows are
// prefetched into that staging with cp.async while the MMA runs and updated in
// place; the QKV epilogue prefetches its tokens' RoPE rows the same way.
//
// Clusters (no load is multicast; partner data crosses by bulk copies into
// the partner's idle operand ring, completing on its mbarrier):
//  - PAIR: two CTAs share each M = 256 tcgen05.mma (cta_group::2), each
//    loading its own 128 rows of A and half of B (opt-in);
//  - csplit (normal orientation, clusters of two): a tile whose k-range
//    stream-K splits exactly between the two CTAs is finished in column
//    halves, each CTA sending the other its half-partial of the other's
//    columns;
//  - cred (swapped, clusters of up to 8): each tile's pieces are the CTAs of
//    one cluster, one equal k-range each; every CTA sends each partner its
//    4-column slice of that partner's token columns and finishes its own,
//    summing the slices in rank (= k) order -- the ticket path's order, so
//    the result is bitwise the same.  Each CTA arrives at the cluster's exit
//    barrier when it is done with its partners and waits there before it
//    leaves, so none leaves while a partner may still copy into it.
//
// Warp roles (192 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA
// issuer, warps 2..5 epilogue (warp w reads TMEM lanes 32*(w%4) .. +31).
#include <cstdio>

#include "common.cuh"
#include "kernels.h"

namespace wam {
static_assert(kRowNormMax == 32 * 4 * kRowNormV, "norm row width limit");
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kThreads = 192;
constexpr int kBox = 4096;  // one output box: 32 rows x 128 bytes

// Epilogue class of a kernel instance: which shared-memory staging it carries.
enum : int {
  kClassScalar = 0,  // per-element stores (Euler update, video endpoint; every swapped epilogue)
  kClassStore = 1,   // fp32 store / GELU: two output boxes per warp
  kClassRes = 2,     // gate-residual: the warp's 32 x BN residual rows (BN <= 128)
  kClassQkv = 3,     // QK-norm + RoPE: 32 cos + 32 sin rows and two output boxes per warp
  kClassNormB = 4,   // swapped, B = RMSNorm/modulation of fp32 token rows computed in the kernel
};

// Largest reduction length of the fused-norm B operand (held whole in shared memory).
constexpr int kNormKMax = 1024;

// PAIR: the CTA is one of a pair sharing an M = 256 MMA (normal orientation):
// it loads its own 128 A rows and half of the tile's BN B rows, and its
// output tile is still 128 x BN.
template <int BN, bool SWAP, int EPI, bool PAIR = false>
struct TileCfg {
  static constexpr bool kNB = EPI == kClassNormB;
  static_assert(!kNB || (SWAP && BN <= 64), "fused-norm B operand: swapped orientation, <= 64 tokens");
  static_assert(!PAIR || (!SWAP && BN == 256 && (EPI == kClassStore || EPI == kClassRes || EPI == kClassQkv)),
                "CTA pairs: normal orientation, 256-wide tiles, TMA-store epilogues");
  static constexpr int kABytes = BM * BK * 2;
  static constexpr int kBRows = PAIR ? BN / 2 : BN;      // B rows this CTA loads
  static constexpr int kBBytes = kNB ? 0 : kBRows * BK * 2;  // per stage
  static constexpr int kStageBytes = kABytes + kBBytes;
  // fused-norm B operand, resident: [k-block][BN rows][128 B], 128-byte swizzle
  static constexpr int kResB = kNB ? (kNormKMax / BK) * BN * 128 : 0;
  static constexpr int kTmemCols = 2 * BN <= 32 ? 32 : (2 * BN <= 64 ? 64 : (2 * BN <= 128 ? 128 : (2 * BN <= 256 ? 256 : 512)));
  // gate-residual: up to 128 columns the warp's whole 32 x BN residual block
  // is prefetched; wider tiles stream it box by box through two buffers
  static constexpr bool kResBoxes = EPI == kClassRes && BN > 128;
  static constexpr int kWarpStg = SWAP ? 0
                                       : (EPI == kClassStore ? 2 * kBox
                                                             : (EPI == kClassRes ? (kResBoxes ? 2 * kBox : 32 * BN * 4)
                                                                                 : (EPI == kClassQkv ? 4 * kBox : 0)));
  static constexpr int kSwapStg = SWAP ? 32 * (BM + 1) * 4 : 0;  // swapped QKV staging [32 tokens][129]
  // the tile's bias slice (and gate or QK gains) in shared memory, normal orientation
  static constexpr int kVecBytes = (SWAP || EPI == kClassScalar) ? 0 : (EPI == kClassStore ? 1 : 2) * BN * 4;
  static constexpr int kExtra = kResB + 4 * kWarpStg + kSwapStg + kVecBytes;
  static constexpr int kBarBytes = 256;
  static constexpr int kSmemMax = 232448;  // 227 KB per CTA
  // no alignment slack: the dynamic shared memory of a kernel without static
  // shared memory starts on a 1024-byte boundary (checked at run time)
  static constexpr int kFit = (kSmemMax - kBarBytes - kExtra) / kStageBytes;
  static constexpr int kStages = kFit > 8 ? 8 : kFit;
  static constexpr int kSmem = kStages * kStageBytes + kExtra + kBarBytes;
  static_assert(kStages >= 3, "shared memory ring too shallow");
};

struct GemmK {
  int rows_a, rows_b, K;
  int z_a, z_b;
  int tiles_a;
  int KB;        // k-blocks per tile
  long long W;   // k-blocks of all tiles
  int G;         // CTAs sharing them
  float* ws;     // [G][2][BM * BN] partial tiles
  int* tickets;  // [tiles][2]: pieces arrived, pieces published
  unsigned* status;
  int csplit;    // launched as clusters of two CTAs: a tile split between them is finished in halves
  int cred;      // swapped: launched as clusters of cred CTAs, each tile's pieces one cluster (one
                 // equal k-range per CTA), summed in shared memory: each CTA finishes BN / cred columns
};

// First k-block of CTA c, and the CTA owning k-block x (the largest c with
// W c / G <= x).
__device__ __forceinline__ long long kbound(const GemmK& g, int c) { return g.W * c / g.G; }
__device__ __forceinline__ int kowner(const GemmK& g, long long x) { return (int)(((x + 1) * g.G - 1) / g.W); }

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Generic-proxy writes to shared memory become visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
// 3-D tiled store shared -> global; out-of-range rows / columns are not written.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Contiguous bulk copy global -> shared completing `bytes` on `bar` (no multicast).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
// Later async-proxy reads of global memory see what this thread has observed.
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// ---- CTA pairs (2-SM MMA): two CTAs of a cluster of two share one M = 256
// tensor-core tile.  Rank 0 issues the MMAs; each CTA holds its 128 A rows
// and half of the B rows at the same shared-memory offsets, and its 128 rows
// of the accumulator in its own TMEM.
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// All threads of both CTAs; orders every earlier memory operation (remote
// mbarrier arrivals included) before anything after it in the other CTA.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// A liveness point split in two: each thread arrives when it is done with
// the other CTAs of the cluster (no memory ordering), and waits before it
// exits until every thread of the cluster has arrived.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait;" ::: "memory"); }
// Address, in the cluster's shared window, of the same object in CTA `rank`.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
  return a;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}
// Bulk copy of `bytes` from this CTA's shared memory to cluster address `dst`
// (another CTA of the cluster), completing on the barrier at cluster address
// `bar` in that CTA (no multicast).
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "r"(smem_u32(src)), "r"(bytes), "r"(bar)
               : "memory");
}
// TMEM allocation of a pair: the same warp of both CTAs, same slot offset.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* slot_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// 3-D tiled load into this CTA's shared memory whose bytes complete on the
// barrier at cluster address `bar` -- a barrier of either CTA of the pair
// (the 2-SM form of the load; no multicast).
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* map, uint32_t bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}
// D (both CTAs' TMEM) (+)= A (both CTAs' rows) * B (both CTAs' halves)^T.
__device__ __forceinline__ void tc_mma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on the barrier at cluster address `addr` (this CTA's or the peer's)
// once every pair MMA issued so far by this thread completes.
__device__ __forceinline__ void tc_commit_pair(uint32_t addr) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(addr)
               : "memory");
}

#ifdef WAM_GEMM_TIMELINE
// Diagnostic build only: per CTA of the last launch, %smid and %globaltimer
// at start, first MMA issue (rank 0 / single CTA), last MMA issue and end.
__device__ unsigned long long g_gemm_tl[1024][16];
#define WAM_TL(slot, v) \
  if (blockIdx.x < 1024) g_gemm_tl[blockIdx.x][slot] = (v)
#else
#define WAM_TL(slot, v)
#endif

}  // namespace
WAM_KTRACE_UNIT(gemm)
namespace {

// Failure-path test hook (wam_test_peer_wait): the last piece of a split tile
// that is its CTA's final segment waits for g_peer_wait_extra more published
// partials than exist, with the limit g_peer_wait_limit_ns, so that the
// bounded wait gives up on a flag nothing sets.  Zero / kWaitLimitNs (the
// defaults) leave the kernel as it is.
__device__ int g_peer_wait_extra = 0;
__device__ unsigned long long g_peer_wait_limit_ns = kWaitLimitNs;

// Bounded wait until *count >= target (a counter other CTAs increment).
__device__ __forceinline__ bool wait_count(const int* count, int target, unsigned* status, volatile int* abort,
                                           unsigned long long limit_ns = kWaitLimitNs) {
  // One polling thread (the rest of its CTA waits at a barrier); each poll is
  // an L2 round trip, so no sleep between polls: a __nanosleep here delayed
  // the split-tile reducer by ~1.7 us after the last partner had published.
  const volatile int* vc = count;
  const unsigned long long t0 = globaltimer();
  while (*vc < target) {
    if (abort && *abort) return false;
    if (globaltimer() - t0 > limit_ns) {
      atomicOr(status, kStatusTimeoutPeer);
      return false;
    }
  }
  return true;
}

// 16-byte chunk q of row r (0..31) of a 32 x 128-byte box: the layout a TMA
// box with the 128-byte swizzle has in shared memory (chunk q at q ^ (r & 7)).
__device__ __forceinline__ uint4* box_chunk(uint8_t* box, int r, int q) {
  return reinterpret_cast<uint4*>(box + r * 128 + ((q ^ (r & 7)) << 4));
}

__device__ __forceinline__ void box_row_f32(uint8_t* box, int r, const float* v) {  // 32 values
#pragma unroll
  for (int q = 0; q < 8; ++q)
    *box_chunk(box, r, q) = make_uint4(__float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]),
                                       __float_as_uint(v[4 * q + 2]), __float_as_uint(v[4 * q + 3]));
}
__device__ __forceinline__ void box_row_bf16(uint8_t* box, int r, const float* v) {  // 64 values
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    uint4 w;
    w.x = pack_bf16(v[8 * q + 0], v[8 * q + 1]);
    w.y = pack_bf16(v[8 * q + 2], v[8 * q + 3]);
    w.z = pack_bf16(v[8 * q + 4], v[8 * q + 5]);
    w.w = pack_bf16(v[8 * q + 6], v[8 * q + 7]);
    *box_chunk(box, r, q) = w;
  }
}

// Epilogue arguments copied into registers once: the store loops never
// re-read the kernel's parameter block (a global store could otherwise force
// a reload of every field after it).
struct EpiRegs {
  int kind;
  const float* bias;
  const float* gate;
  float* out_f32;
  __nv_bfloat16* out_act;
  int ld;
  const float* gq;
  const float* gk;
  const float* rope_cos;
  const float* rope_sin;
  __nv_bfloat16* q_out;
  __nv_bfloat16* k_cache;
  __nv_bfloat16* v_cache;
  int seq_len, cache_len, cache_off, n_heads, attn_dim;
  int zq0, zk0, zv0;
};

__device__ __forceinline__ EpiRegs hoist(const EpiArgs& e) {
  EpiRegs r;
  r.kind = e.kind;
  r.bias = e.bias;
  r.gate = e.gate;
  r.out_f32 = e.out_f32;
  r.out_act = reinterpret_cast<__nv_bfloat16*>(e.out_act);
  r.ld = e.ld_out;
  r.gq = e.gq;
  r.gk = e.gk;
  r.rope_cos = e.rope_cos;
  r.rope_sin = e.rope_sin;
  r.q_out = reinterpret_cast<__nv_bfloat16*>(e.q_out);
  r.k_cache = reinterpret_cast<__nv_bfloat16*>(e.k_cache);
  r.v_cache = reinterpret_cast<__nv_bfloat16*>(e.v_cache);
  r.seq_len = e.seq_len;
  r.cache_len = e.cache_len;
  r.cache_off = e.cache_off;
  r.n_heads = e.n_heads;
  r.attn_dim = e.attn_dim;
  r.zq0 = e.zq0;
  r.zk0 = e.zk0;
  r.zv0 = e.zv0;
  return r;
}

// Per-head QK-RMSNorm (gain) and RoPE of the 64-channel head vector x of
// token m (section 0 = q, 1 = k; 2 = v is left as is).  cs_row / sn_row: the
// token's cos / sin row in shared memory with 16-byte chunk q at q ^ swz, or
// null to read the tables.
__device__ __forceinline__ void qk_norm_rope(const EpiRegs& R, int section, int head, int m, float (&x)[64],
                                             const float* cs_row, const float* sn_row, int swz,
                                             const float* gain = nullptr) {
  if (section >= 2) return;
  const int l = m % R.seq_len;
  const float4* g4 = reinterpret_cast<const float4*>(gain ? gain : (section == 0 ? R.gq : R.gk) + head * 64);
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < 64; ++j) ss += x[j] * x[j];
  const float r = rsqrtf(ss * (1.0f / 64.0f) + 1e-6f);
#pragma unroll
  for (int j4 = 0; j4 < 16; ++j4) {
    const float4 gg = gain ? g4[j4] : __ldg(g4 + j4);
    x[4 * j4] *= r * gg.x;
    x[4 * j4 + 1] *= r * gg.y;
    x[4 * j4 + 2] *= r * gg.z;
    x[4 * j4 + 3] *= r * gg.w;
  }
  const int pos = R.cache_off + l;
  const float4* cs = reinterpret_cast<const float4*>(cs_row ? cs_row : R.rope_cos + pos * 32);
  const float4* sn = reinterpret_cast<const float4*>(sn_row ? sn_row : R.rope_sin + pos * 32);
#pragma unroll
  for (int j4 = 0; j4 < 8; ++j4) {
    const float4 c4 = cs[cs_row ? (j4 ^ swz) : j4], s4 = sn[sn_row ? (j4 ^ swz) : j4];
    const float cc[4] = {c4.x, c4.y, c4.z, c4.w}, ss4[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = 4 * j4 + q;
      const float x1 = x[j], x2 = x[j + 32];
      x[j] = x1 * cc[q] - x2 * ss4[q];
      x[j + 32] = x1 * ss4[q] + x2 * cc[q];
    }
  }
}

// Global row of token m, head `head` in Q (section 0) or the K / V cache.
__device__ __forceinline__ __nv_bfloat16* qkv_dst(const EpiRegs& R, int section, int head, int m) {
  const int b = m / R.seq_len, l = m - b * R.seq_len;
  if (section == 0) return R.q_out + ((size_t)(b * R.n_heads + head) * R.seq_len + l) * 64;
  return (section == 1 ? R.k_cache : R.v_cache) + ((size_t)(b * R.n_heads + head) * R.cache_len + R.cache_off + l) * 64;
}

__device__ __forceinline__ void store_head(__nv_bfloat16* dst, const float (&x)[64]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    uint4 w;
    w.x = pack_bf16(x[8 * j + 0], x[8 * j + 1]);
    w.y = pack_bf16(x[8 * j + 2], x[8 * j + 3]);
    w.z = pack_bf16(x[8 * j + 4], x[8 * j + 5]);
    w.w = pack_bf16(x[8 * j + 6], x[8 * j + 7]);
    d4[j] = w;
  }
}

// Elementwise epilogue of one value at (token m, feature n) with y = acc + bias[n].
__device__ __forceinline__ void epi_elem(const EpiArgs& e, int m, int n, float y, float gate) {
  const size_t idx = (size_t)m * e.ld_out + n;
  switch (e.kind) {
    case kEpiStoreF32:
      e.out_f32[idx] = y;
      break;
    case kEpiGateRes:
      e.out_f32[idx] += gate * y;
      break;
    case kEpiGelu:
      reinterpret_cast<__nv_bfloat16*>(e.out_act)[idx] = __float2bfloat16_rn(gelu_tanh(y));
      break;
    case kEpiScaleAct:
      reinterpret_cast<__nv_bfloat16*>(e.out_act)[idx] = __float2bfloat16_rn(e.scale * y);
      break;
    case kEpiEuler: {
      const float dt = e.aio->sched[e.step] - e.aio->sched[e.step + 1];
      const float a = e.out_f32[idx] - dt * y;
      e.out_f32[idx] = a;
      if (e.a_next) reinterpret_cast<__nv_bfloat16*>(e.a_next)[(size_t)m * e.a_next_ld + n] = __float2bfloat16_rn(a);
      break;
    }
    case kEpiVideoOut: {
      const float sigma = e.vio->t;
      const float s2 = sigma * sigma;
      const float cs = 0.25f / (s2 + 0.25f), co = sigma * 0.5f / sqrtf(s2 + 0.25f);
      const float xs = e.x_sigma[idx];
      e.vio->video_out[idx] = cs * xs + co * (xs - sigma * y);
      break;
    }
    case kEpiVideoEuler: {
      const float ds = e.vio->vsched[e.step] - e.vio->vsched[e.step + 1];
      const float xn = e.out_f32[idx] - ds * y;
      e.out_f32[idx] = xn;
      if (e.out_act) reinterpret_cast<__nv_bfloat16*>(e.out_act)[(size_t)m * e.a_next_ld + n] = __float2bfloat16_rn(xn);
      if (e.step == e.vio->vsteps - 1) e.vio->video_out[idx] = xn;
      break;
    }
    default:
      break;
  }
}

// The next segment of a CTA's k-block range starting at x: tile t, k-blocks
// [kb0, kb1) of it.
struct Seg {
  int t, kb0, kb1;
};
__device__ __forceinline__ Seg seg_at(const GemmK& g, long long x, long long x_end) {
  Seg s;
  s.t = (int)(x / g.KB);
  s.kb0 = (int)(x - (long long)s.t * g.KB);
  const long long lim = s.kb0 + (x_end - x);
  s.kb1 = lim < g.KB ? (int)lim : g.KB;
  return s;
}

template <int BN, bool SWAP, int EPI, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                   const __grid_constant__ CUtensorMap map_o, const __grid_constant__ CUtensorMap map_o2,
                   const GemmK g, const EpiArgs e) {
  using C = TileCfg<BN, SWAP, EPI, PAIR>;
  WAM_KT_BEGIN;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // The 128-byte swizzle is a function of the address bits: every tile must
  // start on a 1024-byte boundary.
  if (smem_u32(smem_raw) & 1023) {
    if (threadIdx.x == 0) atomicOr(g.status, kStatusTimeoutDrain);
    return;
  }
#ifdef WAM_GEMM_TIMELINE
  if (threadIdx.x == 0) {
    unsigned sm;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
    WAM_TL(0, sm);
    WAM_TL(1, globaltimer());
  }
#endif
  uint8_t* smem = smem_raw;
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::kStages * C::kABytes;
  uint8_t* sBres = smem + C::kStages * C::kStageBytes;  // fused-norm B operand (1024-byte aligned)
  uint8_t* sStg = sBres + C::kResB;                     // epilogue staging (1024-byte aligned)
  float* sVec = reinterpret_cast<float*>(sStg + 4 * C::kWarpStg + C::kSwapStg);  // [BN] bias, [BN] gate / gains
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes + C::kExtra);
  uint64_t* empty = full + C::kStages;
  uint64_t* accf = empty + C::kStages;  // [2] accumulator ready (MMA -> epilogue)
  uint64_t* acce = accf + 2;            // [2] accumulator drained (epilogue -> MMA)
  uint64_t* redb = acce + 2;            // partial tiles copied into the ring
  uint64_t* bready = redb + 1;          // fused-norm B operand written (epilogue warps -> MMA)
  uint64_t* peer_idle = bready + 1;     // cluster split / reduce: the partners' rings may take my partials
  uint64_t* peer_data = peer_idle + 1;  // cluster split / reduce: the partners' partials are in my ring
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(peer_data + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Stream-K unit: the CTA, or the CTA pair (both CTAs of a pair run the same
  // segments; rank 1 takes the odd 128-row tile of each 256-row pair tile).
  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  bool cl_arrived = false;  // cluster reduce: this thread has arrived at the exit barrier
  const long long x_begin = kbound(g, unit), x_end = kbound(g, unit + 1);

  if (threadIdx.x == 0) {
    // rank 0 of a pair: an accumulator is drained once both CTAs'
    // epilogues are done (the peer's stage bytes complete on rank 0's full
    // barriers, which expect both CTAs' bytes)
    const bool lead = PAIR && rank == 0;
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], lead ? 8 : 4);
    }
    mbar_init(redb, 1);
    mbar_init(bready, 1);
    mbar_init(peer_idle, g.cred > 1 ? g.cred - 1 : 1);
    mbar_init(peer_data, 1);
    *abort_flag = 0;
    *last_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&map_a);
    if (!C::kNB) prefetch_tensormap(&map_b);
    if (!SWAP && EPI != kClassScalar) prefetch_tensormap(&map_o);
    if (!SWAP && EPI == kClassQkv) prefetch_tensormap(&map_o2);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, C::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, C::kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();  // the peer's barriers exist before any remote arrival
  if (!PAIR && (g.csplit || g.cred > 1)) cluster_sync();  // (the same for the cluster split / reduce; g is uniform)
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();  // the next kernel may start its own set-up now

  // first rows of this CTA's A and B loads for tile (ta, tb)
  auto arow = [&](int ta) { return SWAP ? ta * BM : (PAIR ? 2 * ta + (int)rank : ta) * BM; };
  auto brow = [&](int tb) { return SWAP ? tb * BN : tb * BN + (PAIR ? (int)rank * C::kBRows : 0); };

  if (warp == 0) {
    if (lane == 0) {
      int it = 0, issued = 0;
      bool ok = true;
      // Stage st's loads.  A pair's stage is one barrier, rank 0's: rank 0
      // arms it for both CTAs' bytes and the peer's loads complete on it.
      const bool peer = PAIR && rank == 1;
      auto arm = [&](int st) {
        if (!peer) mbar_arrive_expect_tx(&full[st], (PAIR ? 2 : 1) * C::kStageBytes);
      };
      auto load = [&](const CUtensorMap* map, uint8_t* dst, int st, int kb, int y, int z) {
        if (peer)
          tma_load_3d_pair(dst, map, cluster_addr(&full[st], 0), kb * BK, y, z);
        else
          tma_load_3d(dst, map, &full[st], kb * BK, y, z);
      };
      // The weights never change during a chunk: the first segment's weight
      // tiles are requested before waiting for the previous kernel.
      int pre = 0;
      if (x_begin < x_end) {
        const Seg sg = seg_at(g, x_begin, x_end);
        const int ta = sg.t % g.tiles_a, tb = sg.t / g.tiles_a;
        pre = min(C::kStages, sg.kb1 - sg.kb0);
        for (int i = 0; i < pre; ++i) {
          arm(i);
          if (SWAP)
            load(&map_a, sA + i * C::kABytes, i, sg.kb0 + i, arow(ta), g.z_a);
          else
            load(&map_b, sB + i * C::kBBytes, i, sg.kb0 + i, brow(tb), g.z_b);
        }
        // with the fused norm the producer reads weights only: no wait for the previous kernel
        if (!C::kNB) pdl_wait();
        WAM_KT_WAITED();
        if (!SWAP && e.na_x) {
          // the A operand is written by this launch (norm prologue): every row done
          if (!wait_count(e.na_cnt + 1, g.rows_a, g.status, abort_flag)) *abort_flag = 1;
          __threadfence();
          fence_proxy_async_global();  // (the loads are issued either way, so every stage completes)
        }
        for (int i = 0; i < pre && !C::kNB; ++i) {
          if (SWAP)
            load(&map_b, sB + i * C::kBBytes, i, sg.kb0 + i, brow(tb), g.z_b);
          else
            load(&map_a, sA + i * C::kABytes, i, sg.kb0 + i, arow(ta), g.z_a);
        }
        issued = pre;
      } else if (!C::kNB) {
        pdl_wait();
      }
      for (long long x = x_begin; x < x_end && ok;) {
        const Seg sg = seg_at(g, x, x_end);
        x += sg.kb1 - sg.kb0;
        const int ta = sg.t % g.tiles_a, tb = sg.t / g.tiles_a;
        for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++it) {
          if (it < pre) continue;  // issued above
          const int s = it % C::kStages;
          if (it >= C::kStages &&
              !mbar_wait(&empty[s], ((it / C::kStages) - 1) & 1, g.status, kStatusTimeoutTmaEmpty, abort_flag)) {
            ok = false;
            break;
          }
          arm(s);
          load(&map_a, sA + s * C::kABytes, s, kb, arow(ta), g.z_a);
          if (!C::kNB) load(&map_b, sB + s * C::kBBytes, s, kb, brow(tb), g.z_b);
          issued = it + 1;
        }
      }
      // Drain: never leave the CTA with copies into its shared memory in
      // flight (a pair's rank 0 waits for both CTAs' bytes; the peer's
      // arrive there) ...
      if (!peer)
        for (int i = max(0, issued - C::kStages); i < issued; ++i)
          mbar_wait(&full[i % C::kStages], (i / C::kStages) & 1, g.status, kStatusTimeoutDrain, nullptr);
      if constexpr (PAIR) {
        // ... nor with the pair's MMAs still reading it: the commits of the
        // last stages have arrived (every issued stage is consumed first;
        // one shared limit for all of them)
        volatile int gave_up = 0;
        for (int i = max(0, issued - C::kStages); i < issued; ++i)
          mbar_wait(&empty[i % C::kStages], (i / C::kStages) & 1, g.status, kStatusTimeoutDrain, &gave_up);
      }
    }
  } else if (warp == 1) {
    if (PAIR && rank == 1) {
      // the peer's MMA warp has nothing to issue: rank 0 runs the pair's MMAs
    } else if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(PAIR ? 2 * BM : BM, BN);
      int it = 0, lt = 0;
      bool ok = true;
      if (C::kNB && x_begin < x_end) {  // the B operand is computed by the epilogue warps
        ok = mbar_wait(bready, 0, g.status, kStatusTimeoutTmaFull, abort_flag);
        tc_fence_after();
      }
      for (long long x = x_begin; x < x_end && ok; ++lt) {
        const Seg sg = seg_at(g, x, x_end);
        x += sg.kb1 - sg.kb0;
        const int buf = lt & 1;
        if (lt >= 2 &&
            !mbar_wait(&acce[buf], ((lt >> 1) - 1) & 1, g.status, kStatusTimeoutAccum, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + buf * BN;
        for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++it) {
          const int s = it % C::kStages;
          if (!mbar_wait(&full[s], (it / C::kStages) & 1, g.status, kStatusTimeoutTmaFull, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (it == 0) WAM_TL(2, globaltimer());
          WAM_TL(3, globaltimer());
          const uint32_t a0 = smem_u32(sA + s * C::kABytes);
          const uint32_t b0 = C::kNB ? smem_u32(sBres + kb * (BN * 128)) : smem_u32(sB + s * C::kBBytes);
          if constexpr (PAIR) {
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              tc_mma_bf16_pair(d_tmem, smem_desc_k128(a0 + k * 32), smem_desc_k128(b0 + k * 32), idesc,
                               (kb > sg.kb0 || k > 0) ? 1u : 0u);
            tc_commit_pair(smem_u32(&empty[s]));  // both CTAs may refill the stage
            tc_commit_pair(cluster_addr(&empty[s], 1));
          } else {
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              tc_mma_bf16(d_tmem, smem_desc_k128(a0 + k * 32), smem_desc_k128(b0 + k * 32), idesc,
                          (kb > sg.kb0 || k > 0) ? 1u : 0u);
            tc_commit(&empty[s]);
          }
        }
        if constexpr (PAIR) {
          tc_commit_pair(smem_u32(&accf[buf]));  // both CTAs' accumulator halves are ready
          tc_commit_pair(cluster_addr(&accf[buf], 1));
        } else {
          tc_commit(&accf[buf]);
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    pdl_wait();  // outputs / residual rows belong to the previous kernel until it is done
    if (!SWAP && e.na_x) {
      // Norm prologue: token rows of the A operand, one per warp at a time,
      // from the launch's shared row counter (no CTA waits for another to
      // start: the running CTAs take every row between them).
      int n = 0;
      while (true) {
        int r = 0;
        if (lane == 0) r = atomicAdd(e.na_cnt, 1);
        r = __shfl_sync(0xffffffffu, r, 0);
        if (r >= g.rows_a) break;
        norm_mod_row<true>(e.na_x + (size_t)r * g.K, reinterpret_cast<__nv_bfloat16*>(e.na_h) + (size_t)r * g.K, g.K,
                           e.na_scale, e.na_shift, nullptr, lane);
        ++n;
      }
      if (n > 0) {
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(e.na_cnt + 1, n);
      }
    }
    const int quad = warp & 3;
    const int row = quad * 32 + lane;  // TMEM lane = tile row
    const EpiRegs R = hoist(e);
    if constexpr (C::kNB) {
      // B = rms(x) * (gain or 1 + scale) + shift as bf16, in the layout a
      // 128-byte-swizzled TMA load of [BN rows][64] would give each k-block.
      // Four threads share a row: first every row's sum of squares over all K
      // (loads issued 24 float4 at a time), then only the k-blocks this CTA's
      // segments read.
      const int K = g.K, n4 = K / 4;
      const int te = threadIdx.x - 64;  // 0..127
      float* sRR = reinterpret_cast<float*>(sStg);  // [BN] 1 / rms (the swapped staging is free until then)
      for (int p = 0; p < BN / 32; ++p) {
        const int r = p * 32 + (te >> 2), part = te & 3;
        const bool valid = r < g.rows_b;
        const float4* xr = reinterpret_cast<const float4*>(e.nb_x + (size_t)(valid ? r : 0) * K);
        float ss = 0.f;
        for (int i0 = 0; i0 < n4 / 4; i0 += 24) {
          float4 v[24];
#pragma unroll
          for (int i = 0; i < 24; ++i) {
            const int k4 = part + 4 * (i0 + i);
            v[i] = (valid && k4 < n4) ? xr[k4] : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int i = 0; i < 24; ++i) ss += v[i].x * v[i].x + v[i].y * v[i].y + v[i].z * v[i].z + v[i].w * v[i].w;
        }
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        ss += __shfl_xor_sync(0xffffffffu, ss, 2);
        if (part == 0) sRR[r] = 1.0f / sqrtf(ss / (float)K + 1e-6f);
      }
      epi_bar();
      unsigned need = 0;  // k-blocks of this CTA's segments (K <= 1024: at most 16)
      for (long long xx = x_begin; xx < x_end;) {
        const Seg sg = seg_at(g, xx, x_end);
        xx += sg.kb1 - sg.kb0;
        for (int kb = sg.kb0; kb < sg.kb1; ++kb) need |= 1u << kb;
      }
      for (int kb = 0; kb < K / BK; ++kb) {
        if (!(need >> kb & 1u)) continue;
        const int c0 = kb * BK + (te & 3) * 16;  // this thread's 16 columns
        float4 mul[4], add[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (e.nb_gain) {
            mul[i] = __ldg(reinterpret_cast<const float4*>(e.nb_gain + c0) + i);
          } else {
            mul[i] = __ldg(reinterpret_cast<const float4*>(e.nb_scale + c0) + i);
            mul[i].x += 1.f;
            mul[i].y += 1.f;
            mul[i].z += 1.f;
            mul[i].w += 1.f;
          }
          add[i] = e.nb_shift ? __ldg(reinterpret_cast<const float4*>(e.nb_shift + c0) + i)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        for (int p = 0; p < BN / 32; ++p) {
          const int r = p * 32 + (te >> 2);
          const bool valid = r < g.rows_b;
          const float4* xr = reinterpret_cast<const float4*>(e.nb_x + (size_t)(valid ? r : 0) * K + c0);
          float4 v[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) v[i] = valid ? xr[i] : make_float4(0.f, 0.f, 0.f, 0.f);
          const float rr = sRR[r];
          uint32_t w[8];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            w[2 * i] = valid ? pack_bf16(v[i].x * rr * mul[i].x + add[i].x, v[i].y * rr * mul[i].y + add[i].y) : 0u;
            w[2 * i + 1] = valid ? pack_bf16(v[i].z * rr * mul[i].z + add[i].z, v[i].w * rr * mul[i].w + add[i].w) : 0u;
          }
          const int q = (te & 3) * 2;  // two 16-byte chunks of the 128-byte row
          uint8_t* rowp = sBres + kb * (BN * 128) + r * 128;
          *reinterpret_cast<uint4*>(rowp + ((q ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
          *reinterpret_cast<uint4*>(rowp + (((q + 1) ^ (r & 7)) << 4)) = make_uint4(w[4], w[5], w[6], w[7]);
        }
      }
      fence_proxy_async_smem();  // generic writes -> visible to the tensor core
      epi_bar();                 // (the staging's 1 / rms values are read; it may be reused)
      if (threadIdx.x == 64) mbar_arrive(bready);
    }
    uint8_t* stg = sStg + quad * C::kWarpStg;  // this warp's staging (normal orientation)
    int nbox = 0;                              // output boxes this warp stored (double-buffer index)
    int lt = 0;
    for (long long x = x_begin; x < x_end; ++lt) {
      const bool first_seg = (x == x_begin);
      const Seg sg = seg_at(g, x, x_end);
      x += sg.kb1 - sg.kb0;
      const int t = sg.t;
      const int ta = t % g.tiles_a, tb = t / g.tiles_a;
      const long long t0 = (long long)t * g.KB;
      const int c_first = kowner(g, t0);
      const int npieces = kowner(g, t0 + g.KB - 1) - c_first + 1;
      const int buf = lt & 1;
      // A tile split in two between the CTAs of a cluster that covers exactly
      // their whole k-ranges (stream-K gave CTAs 2k and 2k + 1 one piece each
      // and nothing else): each CTA finishes half of the columns, the
      // partner's half-partial arriving in its idle ring through the
      // cluster's shared window.  Both CTAs decide this alike from g and t.
      const bool cs = !SWAP && !PAIR && C::kStages * C::kStageBytes >= BM * BN * 4 && g.csplit && npieces == 2 &&
                      (c_first & 1) == 0 && kbound(g, c_first) == t0 && kbound(g, c_first + 2) == t0 + g.KB;
      const int c_lo = cs ? (unit - c_first) * (BN / 2) : 0;
      const int c_hi = cs ? c_lo + BN / 2 : BN;
      // A swapped tile whose g.cred pieces are exactly the CTAs of one cluster
      // (each CTA one whole equal k-range): CTA rank rk finishes token columns
      // [rk cw, rk cw + cw), the other pieces' slices of them arriving in its
      // idle ring through the cluster's shared window.  Decided alike by all.
      const bool cr = SWAP && !PAIR && g.cred > 1 && npieces == g.cred && c_first % g.cred == 0 &&
                      kbound(g, c_first) == t0 && kbound(g, c_first + g.cred) == t0 + g.KB;
      const int cw = cr ? BN / g.cred : BN, rk = cr ? unit - c_first : 0;
      // swapped: this thread's feature's bias and gate, and for a cluster
      // reduction with a gate-residual its residual values (when it finishes
      // at most 16 columns), requested now so that they arrive while the
      // MMAs run
      const int n_sw = ta * BM + row;
      const bool n_sw_ok = SWAP && n_sw < g.rows_a;
      const float bias_sw = n_sw_ok ? __ldg(R.bias + n_sw) : 0.f;
      const float gate_sw = (n_sw_ok && R.gate) ? __ldg(R.gate + n_sw) : 0.f;
      float xo_cr[16];
      const bool xo_pf = cr && n_sw_ok && R.kind == kEpiGateRes && cw <= 16;
      if (xo_pf) {
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int m = tb * BN + rk * cw + k;
          xo_cr[k] = k < cw && m < g.rows_b ? R.out_f32[(size_t)m * R.ld + n_sw] : 0.f;
        }
      }
      const int m0w = arow(ta) + quad * 32;  // normal orientation: this warp's first row
      const int tk = PAIR ? 2 * t + (int)rank : t;  // the tickets of this CTA's 128-row tile
      const int nb = tb * BN;

      // ---- prefetch while the MMA of this segment runs
      bool prefetched = false;
      if constexpr (C::kVecBytes > 0) {
        // every warp is done with the previous segment's vectors
        epi_bar();
        if (quad == 0) {
          for (int q4 = lane; q4 < BN / 4; q4 += 32) {
            const int n = nb + 4 * q4;
            const bool v = n < g.rows_b;
            cp_async16(smem_u32(sVec + 4 * q4), v ? (const void*)(R.bias + n) : (const void*)R.bias, v);
            if constexpr (EPI == kClassRes) {
              cp_async16(smem_u32(sVec + BN + 4 * q4), v ? (const void*)(R.gate + n) : (const void*)R.gate, v);
            } else if constexpr (EPI == kClassQkv) {
              // gain of column n: q or k RMSNorm gain of its head channel; v columns take none
              const int section = n / R.attn_dim;
              const float* gsrc = section == 0 ? R.gq : R.gk;
              const bool gv = v && section < 2;
              cp_async16(smem_u32(sVec + BN + 4 * q4), gv ? (const void*)(gsrc + n % R.attn_dim) : (const void*)R.gq,
                         gv);
            }
          }
          cp_async_commit();
          prefetched = true;
        }
      }
      if constexpr (!SWAP && (EPI == kClassRes || EPI == kClassQkv)) {
        if (lane == 0) bulk_wait_read<0>();  // earlier stores have left the staging
        __syncwarp();
        if constexpr (C::kResBoxes) {
          // residual boxes 0 and 1 (columns [c_lo, c_lo + 64)); later boxes
          // stream in during the epilogue
          for (int k = lane; k < 32 * 16; k += 32) {
            const int r = k >> 4, q4 = k & 15;
            const int m = m0w + r, n = nb + c_lo + 4 * q4;
            const bool v = m < g.rows_a && n < g.rows_b;
            cp_async16(smem_u32(box_chunk(stg + (q4 >> 3) * kBox, r, q4 & 7)),
                       v ? (const void*)(R.out_f32 + (size_t)m * R.ld + n) : (const void*)R.out_f32, v);
          }
        } else if constexpr (EPI == kClassRes) {
          // residual rows; box b holds columns [32 b, 32 b + 32) in the store layout
          for (int k = lane; k < 32 * (BN / 4); k += 32) {
            const int r = k / (BN / 4), q4 = k % (BN / 4);
            const int m = m0w + r, n = nb + 4 * q4;
            const bool v = m < g.rows_a && n < g.rows_b;
            cp_async16(smem_u32(box_chunk(stg + (q4 >> 3) * kBox, r, q4 & 7)),
                       v ? (const void*)(R.out_f32 + (size_t)m * R.ld + n) : (const void*)R.out_f32, v);
          }
        } else {
          // cos rows of the warp's 32 tokens at [0, 4 KB), sin rows at [4 KB, 8 KB)
          for (int k = lane; k < 32 * 16; k += 32) {
            const int r = k >> 4, which = (k >> 3) & 1, c4 = k & 7;
            const int m = min(m0w + r, g.rows_a - 1);
            const int pos = R.cache_off + (m % R.seq_len);
            const float* src = (which ? R.rope_sin : R.rope_cos) + pos * 32 + 4 * c4;
            cp_async16(smem_u32(box_chunk(stg + which * kBox, r, c4)), src, true);
          }
        }
        cp_async_commit();
        prefetched = true;
      }

      const bool ok = mbar_wait(&accf[buf], (lt >> 1) & 1, g.status, kStatusTimeoutAccum, abort_flag);
      if (prefetched) {
        cp_async_wait<0>();
        __syncwarp();
      }
      tc_fence_after();
      if (!ok) *abort_flag = 1;
      // one decision for all four epilogue warps (every named barrier below is
      // reached by all of them or by none)
      epi_bar();
      if (*abort_flag) break;
      const uint32_t t_row = tmem + (static_cast<uint32_t>(quad * 32) << 16) + buf * BN;
      auto release = [&]() {  // this warp's TMEM reads of the buffer are done
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (PAIR && rank == 1)
            mbar_arrive_cluster(cluster_addr(&acce[buf], 0));  // the MMAs are issued by rank 0
          else
            mbar_arrive(&acce[buf]);
        }
      };

      if (threadIdx.x == 64 && x == x_end) WAM_TL(5, globaltimer());  // last segment's accumulator ready
      if (cs) {
        // My ring is idle (this segment's MMAs are done, nothing in flight).
        // Its first half receives the partner's half-partial of my columns,
        // its second half stages mine of the partner's columns, both as
        // [32-column chunk][row][32 floats] with the 16-byte chunks of a row
        // rotated by (row & 7) (conflict-free shared-memory access).
        constexpr uint32_t kHalf = BM * (BN / 2) * 4;
        const uint32_t peer = (uint32_t)((unit - c_first) ^ 1);
        if (threadIdx.x == 64) {
          mbar_arrive_expect_tx(peer_data, kHalf);  // what the partner will send
          mbar_arrive_cluster(cluster_addr(peer_idle, peer));  // it may send now
        }
        const int o_lo = BN / 2 - c_lo;  // the partner's columns
        uint8_t* stage = smem + kHalf;
        for (int c = 0; c < BN / 2; c += 32) {
          float v[32];
          tmem_ld32(t_row + o_lo + c, v);
          uint8_t* d = stage + ((c >> 5) * BM + row) * 128;
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(d + ((q ^ (row & 7)) << 4)) =
                make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
        fence_proxy_async_smem();  // generic writes -> the bulk copy
        epi_bar();
        if (threadIdx.x == 64) {
          if (!mbar_wait(peer_idle, 0, g.status, kStatusTimeoutPeer, abort_flag)) {
            *abort_flag = 1;
          } else {
            bulk_copy_to_peer(cluster_addr(smem, peer), stage, kHalf, cluster_addr(peer_data, peer));
            bulk_commit();
          }
        }
        if (!mbar_wait(peer_data, 0, g.status, kStatusTimeoutPeer, abort_flag)) *abort_flag = 1;
        if (threadIdx.x == 64) bulk_wait_read<0>();  // my staging has been read out (before it is reused)
        epi_bar();
        if (threadIdx.x == 64 && x == x_end) WAM_TL(6, globaltimer());  // exchange done
        if (*abort_flag) break;
      }
      if (cr) {
        // My ring is idle (my one piece's MMAs are done, nothing in flight).
        // Its front holds every piece's slice of my columns, [src rank][4-
        // column chunk][row] float4: mine written here, the others' arriving
        // by bulk copy; behind it I stage my slices of the others' columns the
        // same way, one contiguous block per destination.
        const int S = g.cred, nq = cw / 4;
        const uint32_t slice = (uint32_t)BM * cw * 4;
        uint8_t* stage = smem + (size_t)S * slice;
        // epilogue thread tt < S - 1 deals with partner q(tt): tells it my ring
        // is idle, later sends it my slice of its columns
        const int tt = threadIdx.x - 64, qt = tt < rk ? tt : tt + 1;
        if (threadIdx.x == 64) mbar_arrive_expect_tx(peer_data, (S - 1) * slice);  // what the others will send
        // (relaxed: nothing to publish -- my MMAs' reads of the ring completed
        // before the accumulator was reported ready)
        if (tt < S - 1) mbar_arrive_cluster_relaxed(cluster_addr(peer_idle, (uint32_t)qt));  // qt may send now
        for (int c = 0; c < BN; c += 32) {
          float v[32];
          tmem_ld32(t_row + c, v);
#pragma unroll
          for (int i4 = 0; i4 < 8; ++i4) {
            const int col = c + 4 * i4, q = col / cw, qq = (col % cw) >> 2;
            uint8_t* dst = q == rk ? smem + ((size_t)(rk * nq + qq) * BM + row) * 16
                                   : stage + ((size_t)((q < rk ? q : q - 1) * nq + qq) * BM + row) * 16;
            *reinterpret_cast<float4*>(dst) = make_float4(v[4 * i4], v[4 * i4 + 1], v[4 * i4 + 2], v[4 * i4 + 3]);
          }
        }
        release();  // the accumulator is in shared memory now
        fence_proxy_async_smem();  // generic writes -> the bulk copies
        epi_bar();
        if (threadIdx.x == 64 && x == x_end) WAM_TL(10, globaltimer());  // staged
        if (tt < S - 1) {
          if (!mbar_wait(peer_idle, 0, g.status, kStatusTimeoutPeer, abort_flag)) {
            *abort_flag = 1;
          } else {
            if (tt == 0 && x == x_end) WAM_TL(11, globaltimer());  // every partner's ring idle
            // my slice of qt's columns (stage slot tt) into qt's ring at my rank's slot
            bulk_copy_to_peer(cluster_addr(smem + (size_t)rk * slice, (uint32_t)qt), stage + (size_t)tt * slice, slice,
                              cluster_addr(peer_data, (uint32_t)qt));
            bulk_commit();
            if (tt == 0 && x == x_end) WAM_TL(12, globaltimer());  // copy issued
          }
        }
        if (!mbar_wait(peer_data, 0, g.status, kStatusTimeoutPeer, abort_flag)) *abort_flag = 1;
        if (threadIdx.x == 64 && x == x_end) WAM_TL(13, globaltimer());  // every partner's slice arrived
        if (tt < S - 1) bulk_wait_read<0>();  // my staging has been read out
        // done with the other CTAs (their slices are here, mine are read out)
        if (!cl_arrived) cluster_arrive_relaxed();
        cl_arrived = true;
        epi_bar();
        if (threadIdx.x == 64 && x == x_end) WAM_TL(6, globaltimer());  // exchange done
        if (*abort_flag) break;
      }
      // ---- a tile shared with other CTAs (see "Split tiles" above)
      const int mine = unit - c_first;  // this CTA's piece of tile t
      // CTA holding piece p's partial (the same rank of the piece's pair)
      auto piece_cta = [&](int p) { return PAIR ? 2 * (c_first + p) + (int)rank : c_first + p; };
      bool from_smem = false;
      if (npieces > 1 && !cs && !cr) {
        if (threadIdx.x == 64) {
          const int prev = atomicAdd(g.tickets + 2 * tk, 1);
          *last_flag = (prev == npieces - 1) ? 1 : 0;
        }
        epi_bar();
        if (*last_flag == 0) {
          // publish: [32-column chunk][j][row][4], a warp's stores contiguous
          float* my = g.ws + ((size_t)blockIdx.x * 2 + (first_seg ? 0 : 1)) * (BM * BN);
          for (int c = 0; c < BN; c += 32) {
            float v[32];
            if (threadIdx.x == 64 && c < 64 && x == x_end) WAM_TL(10 + 3 * (c >> 5), globaltimer());
            tmem_ld32(t_row + c, v);
            if (threadIdx.x == 64 && c < 64 && x == x_end) WAM_TL(11 + 3 * (c >> 5), globaltimer());
            if (c + 32 >= BN) release();
#pragma unroll
            for (int j = 0; j < 8; ++j)
              __stcg(reinterpret_cast<float4*>(my + ((size_t)((c >> 5) * 8 + j) * BM + row) * 4),
                     make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
            if (threadIdx.x == 64 && c < 64 && x == x_end) WAM_TL(12 + 3 * (c >> 5), globaltimer());
          }
          __threadfence();
          epi_bar();
          if (threadIdx.x == 64) atomicAdd(g.tickets + 2 * tk + 1, 1);
          if (threadIdx.x == 64 && x == x_end) WAM_TL(9, globaltimer());  // published (not the reducer)
          continue;
        }
        // the last arrival reduces: the others have arrived; wait until they have published
        if (threadIdx.x == 64) {
          const bool hooked = x == x_end && g_peer_wait_extra > 0;
          if (!wait_count(g.tickets + 2 * tk + 1, npieces - 1 + (hooked ? g_peer_wait_extra : 0), g.status, abort_flag,
                          hooked ? g_peer_wait_limit_ns : kWaitLimitNs)) {
            *abort_flag = 1;
          } else {
            g.tickets[2 * tk] = 0;  // every piece is done with the tickets
            g.tickets[2 * tk + 1] = 0;
            __threadfence();
            constexpr uint32_t kPart = BM * BN * 4;
            if (x == x_end && (uint32_t)(npieces - 1) * kPart <= (uint32_t)(C::kStages * C::kStageBytes)) {
              // the CTA's last segment: its MMAs are done and the ring is free
              fence_proxy_async_global();
              mbar_arrive_expect_tx(redb, (npieces - 1) * kPart);
              int k = 0;
              for (int p = 0; p < npieces; ++p) {
                if (p == mine) continue;
                const int cp = c_first + p;
                const int slot = (p == 0 && t0 != kbound(g, cp)) ? 1 : 0;
                const uint8_t* src =
                    reinterpret_cast<const uint8_t*>(g.ws + ((size_t)piece_cta(p) * 2 + slot) * (BM * BN));
                for (uint32_t o = 0; o < kPart; o += 32768)
                  bulk_load(smem + k * kPart + o, src + o, min(32768u, kPart - o), redb);
                ++k;
              }
              *last_flag = 2;
            }
          }
        }
        epi_bar();
        if (*abort_flag) break;
        if (threadIdx.x == 64 && x == x_end) WAM_TL(6, globaltimer());  // partners published (reducer)
        from_smem = *last_flag == 2;
        if (from_smem) {
          // at most one bulk reduction per CTA (its last segment): phase 0
          // (no early exit: the copies must land before the CTA may end)
          if (!mbar_wait(redb, 0, g.status, kStatusTimeoutPeer, nullptr)) *abort_flag = 1;
          epi_bar();
          if (*abort_flag) break;
        }
        __threadfence();
      }
      // columns [c, c + 32) of this thread's row: the accumulator, or the sum of
      // all pieces in k order with this CTA's own piece read from TMEM
      auto get = [&](int c, float* v) {
        if (cs) {  // my piece from TMEM + the partner's, in my ring (two pieces: the order is immaterial)
          tmem_ld32(t_row + c, *reinterpret_cast<float(*)[32]>(v));
          if (c + 32 >= c_hi) release();
          const uint8_t* rp = smem + ((size_t)((c - c_lo) >> 5) * BM + row) * 128;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 p4 = *reinterpret_cast<const float4*>(rp + ((q ^ (row & 7)) << 4));
            v[4 * q] += p4.x;
            v[4 * q + 1] += p4.y;
            v[4 * q + 2] += p4.z;
            v[4 * q + 3] += p4.w;
          }
          return;
        }
        if (npieces == 1) {
          tmem_ld32(t_row + c, *reinterpret_cast<float(*)[32]>(v));
          if (c + 32 >= BN) release();
          return;
        }
        float own[32];
        tmem_ld32(t_row + c, own);
        if (c + 32 >= BN) release();
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
        int k = 0;
        for (int p = 0; p < npieces; ++p) {
          if (p == mine) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] += own[i];
            continue;
          }
          float4 t4[8];
          const size_t off = ((size_t)((c >> 5) * 8) * BM + row) * 4;
          if (from_smem) {
            const float* src = reinterpret_cast<const float*>(smem) + (size_t)k * (BM * BN) + off;
#pragma unroll
            for (int j = 0; j < 8; ++j) t4[j] = *reinterpret_cast<const float4*>(src + (size_t)j * BM * 4);
          } else {
            const int cp = c_first + p;
            const int slot = (p == 0 && t0 != kbound(g, cp)) ? 1 : 0;
            const float* src = g.ws + ((size_t)piece_cta(p) * 2 + slot) * (BM * BN) + off;
#pragma unroll
            for (int j = 0; j < 8; ++j) t4[j] = __ldcg(reinterpret_cast<const float4*>(src + (size_t)j * BM * 4));
          }
          ++k;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            v[4 * j] += t4[j].x;
            v[4 * j + 1] += t4[j].y;
            v[4 * j + 2] += t4[j].z;
            v[4 * j + 3] += t4[j].w;
          }
        }
      };

      if constexpr (!SWAP) {
        const int m = m0w + lane;
        const bool warp_rows = m0w < g.rows_a;  // the warp has a valid row
        if constexpr (EPI == kClassStore) {
          const bool gelu = R.kind == kEpiGelu;
          const int cols = gelu ? 64 : 32;  // one 128-byte box row
          for (int c = c_lo; c < c_hi; c += cols) {
            float v[64];
            get(c, v);
            if (gelu) get(c + 32, v + 32);
            if (!warp_rows || nb + c >= g.rows_b) continue;
            const float4* b4 = reinterpret_cast<const float4*>(sVec + c);
            uint8_t* box = stg + (nbox & 1) * kBox;
            if (nbox >= 2) {  // this buffer's previous store has been read out
              if (lane == 0) bulk_wait_read<1>();
              __syncwarp();
            }
            if (gelu) {
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const float4 bb = b4[j];
                v[4 * j] = gelu_tanh(v[4 * j] + bb.x);
                v[4 * j + 1] = gelu_tanh(v[4 * j + 1] + bb.y);
                v[4 * j + 2] = gelu_tanh(v[4 * j + 2] + bb.z);
                v[4 * j + 3] = gelu_tanh(v[4 * j + 3] + bb.w);
              }
              box_row_bf16(box, lane, v);
            } else {
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const float4 bb = b4[j];
                v[4 * j] += bb.x;
                v[4 * j + 1] += bb.y;
                v[4 * j + 2] += bb.z;
                v[4 * j + 3] += bb.w;
              }
              box_row_f32(box, lane, v);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(&map_o, box, nb + c, m0w, 0);
              bulk_commit();
            }
            ++nbox;
          }
        } else if constexpr (EPI == kClassRes) {
          const int nvb = (min(c_hi, g.rows_b - nb) - c_lo) / 32;  // boxes with valid columns in [c_lo, c_hi)
          // box bi's residual rows into buffer bi & 1 (one cp.async group)
          auto load_box = [&](int bi) {
            uint8_t* dst = stg + (bi & 1) * kBox;
            for (int k = lane; k < 32 * 8; k += 32) {
              const int r = k >> 3, q = k & 7;
              const int m = m0w + r, n = nb + c_lo + 32 * bi + 4 * q;
              const bool v = m < g.rows_a;
              cp_async16(smem_u32(box_chunk(dst, r, q)),
                         v ? (const void*)(R.out_f32 + (size_t)m * R.ld + n) : (const void*)R.out_f32, v);
            }
            cp_async_commit();
          };
          for (int c = c_lo; c < c_hi; c += 32) {
            const int bi = (c - c_lo) >> 5;  // box index within this CTA's columns
            float v[32];
            get(c, v);
            if (!warp_rows || nb + c >= g.rows_b) continue;
            if constexpr (C::kResBoxes) {
              if (bi >= 2) {  // loaded at the end of iteration bi - 2; bi + 1 may be in flight
                if (bi + 1 < nvb)
                  cp_async_wait<1>();
                else
                  cp_async_wait<0>();
                __syncwarp();
              }
            }
            uint8_t* box = stg + (C::kResBoxes ? (bi & 1) : (c >> 5)) * kBox;  // the residual of these columns
            const float4* b4 = reinterpret_cast<const float4*>(sVec + c);
            const float4* g4 = reinterpret_cast<const float4*>(sVec + BN + c);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              uint4* p = box_chunk(box, lane, q);
              const uint4 xo = *p;
              const float4 bb = b4[q], gg = g4[q];
              *p = make_uint4(__float_as_uint(__uint_as_float(xo.x) + gg.x * (v[4 * q] + bb.x)),
                              __float_as_uint(__uint_as_float(xo.y) + gg.y * (v[4 * q + 1] + bb.y)),
                              __float_as_uint(__uint_as_float(xo.z) + gg.z * (v[4 * q + 2] + bb.z)),
                              __float_as_uint(__uint_as_float(xo.w) + gg.w * (v[4 * q + 3] + bb.w)));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(&map_o, box, nb + c, m0w, 0);
              bulk_commit();
            }
            if constexpr (C::kResBoxes) {
              if (bi + 2 < nvb) {  // the buffer is free once this store has read it
                if (lane == 0) bulk_wait_read<0>();
                __syncwarp();
                load_box(bi + 2);
              }
            }
          }
        } else if constexpr (EPI == kClassQkv) {
          // all 32 tokens valid and in one sample: one TMA store per head
          const bool whole = m0w + 32 <= g.rows_a && (m0w % R.seq_len) + 32 <= R.seq_len;
          for (int c = c_lo; c < c_hi; c += 64) {
            float x[64];
            get(c, x);
            get(c + 32, x + 32);
            const int n = nb + c;
            if (!warp_rows || n >= g.rows_b) continue;
            const float4* b4 = reinterpret_cast<const float4*>(sVec + c);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float4 bb = b4[j];
              x[4 * j] += bb.x;
              x[4 * j + 1] += bb.y;
              x[4 * j + 2] += bb.z;
              x[4 * j + 3] += bb.w;
            }
            const int section = n / R.attn_dim, head = (n % R.attn_dim) / 64;
            qk_norm_rope(R, section, head, min(m, g.rows_a - 1), x, reinterpret_cast<const float*>(stg + lane * 128),
                         reinterpret_cast<const float*>(stg + kBox + lane * 128), lane & 7, sVec + BN + c);
            if (whole) {
              uint8_t* box = stg + (2 + (nbox & 1)) * kBox;
              if (nbox >= 2) {
                if (lane == 0) bulk_wait_read<1>();
                __syncwarp();
              }
              box_row_bf16(box, lane, x);
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                const int b = m0w / R.seq_len, l0 = m0w - b * R.seq_len;
                const int bh = b * R.n_heads + head;
                if (section == 0)
                  tma_store_3d(&map_o, box, 0, l0, R.zq0 + bh);
                else
                  tma_store_3d(&map_o2, box, 0, R.cache_off + l0, (section == 1 ? R.zk0 : R.zv0) + bh);
                bulk_commit();
              }
              ++nbox;
            } else if (m < g.rows_a) {
              store_head(qkv_dst(R, section, head, m), x);
            }
          }
        } else {
          // per-element epilogue (Euler update, video endpoint)
          for (int c = c_lo; c < c_hi; c += 32) {
            float v[32];
            get(c, v);
            const int n0 = nb + c;
            if (m >= g.rows_a || n0 >= g.rows_b) continue;
            const float4* b4 = reinterpret_cast<const float4*>(R.bias + n0);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float4 bb = __ldg(b4 + j);
              v[4 * j] += bb.x;
              v[4 * j + 1] += bb.y;
              v[4 * j + 2] += bb.z;
              v[4 * j + 3] += bb.w;
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) epi_elem(e, m, n0 + j, v[j], 0.f);
          }
        }
      } else {
        // swapped: TMEM lane = feature n, column = token
        const int n = ta * BM + row;
        const int mb = tb * BN;
        const bool n_ok = n < g.rows_a;
        const float bias = bias_sw, gate = gate_sw;
        if (cr && R.kind == kEpiQkv) {
          // my token columns summed in rank order, staged [token][128 features
          // + 1], then (token, head) items as in the whole-tile path below
          const float4* rv = reinterpret_cast<const float4*>(smem);
          float* stage = reinterpret_cast<float*>(sStg);
          epi_bar();  // (the stage's previous readers are done)
#pragma unroll
          for (int qq = 0; qq < 8; ++qq) {
            if (qq >= cw / 4) break;
            float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int p = 0; p < g.cred; ++p) {
              const float4 t4 = rv[(size_t)(p * (cw / 4) + qq) * BM + row];
              a.x += t4.x;
              a.y += t4.y;
              a.z += t4.z;
              a.w += t4.w;
            }
            stage[(4 * qq + 0) * (BM + 1) + row] = a.x + bias;
            stage[(4 * qq + 1) * (BM + 1) + row] = a.y + bias;
            stage[(4 * qq + 2) * (BM + 1) + row] = a.z + bias;
            stage[(4 * qq + 3) * (BM + 1) + row] = a.w + bias;
          }
          epi_bar();
          const int tt = threadIdx.x - 64;
          if (tt < 2 * cw) {
            const int j = tt % cw, hh = tt / cw;
            const int m = mb + rk * cw + j;
            const int n0 = ta * BM + hh * 64;
            if (m < g.rows_b && n0 < g.rows_a) {
              float xv[64];
#pragma unroll
              for (int k = 0; k < 64; ++k) xv[k] = stage[j * (BM + 1) + hh * 64 + k];
              const int section = n0 / R.attn_dim, head = (n0 % R.attn_dim) / 64;
              qk_norm_rope(R, section, head, m, xv, nullptr, nullptr, 0);
              store_head(qkv_dst(R, section, head, m), xv);
            }
          }
        } else if (cr) {
          // my token columns [rk cw, rk cw + cw): every piece's slice of them,
          // summed in rank (= k) order, 4 columns at a time
          const float4* rv = reinterpret_cast<const float4*>(smem);
#pragma unroll
          for (int qq = 0; qq < 8; ++qq) {  // cw = BN / cred <= 32
            if (qq >= cw / 4) break;
            float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int p = 0; p < g.cred; ++p) {
              const float4 t4 = rv[(size_t)(p * (cw / 4) + qq) * BM + row];
              a.x += t4.x;
              a.y += t4.y;
              a.z += t4.z;
              a.w += t4.w;
            }
            if (!n_ok) continue;
            const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int e4 = 0; e4 < 4; ++e4) {
              const int m = mb + rk * cw + 4 * qq + e4;
              if (m >= g.rows_b) continue;
              const float y = av[e4] + bias;
              float* o32 = R.out_f32 + (size_t)m * R.ld + n;
              if (R.kind == kEpiGateRes)
                *o32 = (xo_pf && qq < 4 ? xo_cr[(4 * qq + e4) & 15] : *o32) + gate * y;
              else if (R.kind == kEpiStoreF32)
                *o32 = y;
              else if (R.kind == kEpiGelu)
                R.out_act[(size_t)m * R.ld + n] = __float2bfloat16_rn(gelu_tanh(y));
              else if (R.kind == kEpiScaleAct)
                R.out_act[(size_t)m * R.ld + n] = __float2bfloat16_rn(e.scale * y);
              else
                epi_elem(e, m, n, y, gate);
            }
          }
        }
        for (int c = 0; c < BN && !cr; c += 32) {
          float v[32];
          get(c, v);
          if (R.kind == kEpiQkv) {
            // stage [32 tokens][128 features + 1] and emit (token, head) items
            float* stage = reinterpret_cast<float*>(sStg);
            epi_bar();  // the previous chunk's readers are done with the stage
#pragma unroll
            for (int j = 0; j < 32; ++j) stage[j * (BM + 1) + row] = v[j] + bias;
            epi_bar();
            const int tt = threadIdx.x - 64;
            if (tt < 64) {
              const int j = tt & 31, hh = tt >> 5;
              const int m = mb + c + j;
              const int n0 = ta * BM + hh * 64;
              if (m < g.rows_b && n0 < g.rows_a) {
                float xv[64];
#pragma unroll
                for (int k = 0; k < 64; ++k) xv[k] = stage[j * (BM + 1) + hh * 64 + k];
                const int section = n0 / R.attn_dim, head = (n0 % R.attn_dim) / 64;
                qk_norm_rope(R, section, head, m, xv, nullptr, nullptr, 0);
                store_head(qkv_dst(R, section, head, m), xv);
              }
            }
          } else if (n_ok && R.kind == kEpiGateRes) {
            float xo[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int m = mb + c + j;
              xo[j] = m < g.rows_b ? R.out_f32[(size_t)m * R.ld + n] : 0.f;
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int m = mb + c + j;
              if (m < g.rows_b) R.out_f32[(size_t)m * R.ld + n] = xo[j] + gate * (v[j] + bias);
            }
          } else if (n_ok && R.kind == kEpiStoreF32) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int m = mb + c + j;
              if (m < g.rows_b) R.out_f32[(size_t)m * R.ld + n] = v[j] + bias;
            }
          } else if (n_ok && R.kind == kEpiGelu) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int m = mb + c + j;
              if (m < g.rows_b) R.out_act[(size_t)m * R.ld + n] = __float2bfloat16_rn(gelu_tanh(v[j] + bias));
            }
          } else if (n_ok && R.kind == kEpiScaleAct) {
            const float sc = e.scale;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int m = mb + c + j;
              if (m < g.rows_b) R.out_act[(size_t)m * R.ld + n] = __float2bfloat16_rn(sc * (v[j] + bias));
            }
          } else if (n_ok && R.kind == kEpiEuler) {
            // the step's dt once, and the 32 state values (distinct rows) all
            // requested before any store: per-element calls reloaded the
            // schedule and read each value after the previous store (the
            // compiler cannot rule out aliasing), a chain of 32 round trips
            const float dt = e.aio->sched[e.step] - e.aio->sched[e.step + 1];
            __nv_bfloat16* const a_next = reinterpret_cast<__nv_bfloat16*>(e.a_next);
            const int a_next_ld = e.a_next_ld;
            float a0[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int m = mb + c + j;
              a0[j] = m < g.rows_b ? R.out_f32[(size_t)m * R.ld + n] : 0.f;
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int m = mb + c + j;
              if (m >= g.rows_b) continue;
              const float a = a0[j] - dt * (v[j] + bias);
              R.out_f32[(size_t)m * R.ld + n] = a;
              if (a_next) a_next[(size_t)m * a_next_ld + n] = __float2bfloat16_rn(a);
            }
          } else if (n_ok) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int m = mb + c + j;
              if (m < g.rows_b) epi_elem(e, m, n, v[j] + bias, gate);
            }
          }
        }
      }
    }
    if (threadIdx.x == 64) WAM_TL(7, globaltimer());  // epilogue loop done
    // the warp's bulk stores are complete before the CTA's shared memory goes away
    if (!SWAP && EPI != kClassScalar && lane == 0) bulk_wait_all();
    if (threadIdx.x == 64) WAM_TL(8, globaltimer());
    __syncwarp();
  }
  // the producer and MMA warps (and any thread not yet arrived) are done with
  // the other CTAs of the cluster
  if (!PAIR && g.cred > 1 && !cl_arrived) cluster_arrive_relaxed();

  // ------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // wait for the last commits of this CTA's MMAs before freeing TMEM
    if (lane == 0) {
      int nseg = 0;
      for (long long x = x_begin; x < x_end; ++nseg) {
        const Seg sg = seg_at(g, x, x_end);
        x += sg.kb1 - sg.kb0;
      }
      for (int l = max(0, nseg - 2); l < nseg; ++l)
        mbar_wait(&accf[l & 1], (l >> 1) & 1, g.status, kStatusTimeoutDrain, nullptr);
    }
    __syncwarp();
  }
  // A pair stays until both CTAs are done: rank 0's MMAs read the peer's
  // shared memory, and each CTA arrives on the other's barriers.  So does a
  // cluster that reduces in shared memory (no CTA leaves while a partner
  // might still copy into it, on any path).
  if constexpr (PAIR) cluster_sync();
  if (!PAIR && g.cred > 1) cluster_wait();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem, C::kTmemCols);
    else
      tmem_dealloc(tmem, C::kTmemCols);
  }
  if (threadIdx.x == 0) WAM_TL(4, globaltimer());
  WAM_KT_END(gemm, (unsigned)(BN * 1000 + SWAP * 100 + EPI * 10 + PAIR + 2 * g.csplit));
  if (!SWAP && e.na_x && threadIdx.x == 0) {
    // every CTA is past its rows and its wait once all have counted out here
    __threadfence();
    if (atomicAdd(e.na_cnt + 2, 1) == (int)gridDim.x - 1) {
      e.na_cnt[0] = 0;
      e.na_cnt[1] = 0;
      e.na_cnt[2] = 0;
      __threadfence();
    }
  }
}

template <int BN, bool SWAP, int EPI, bool PAIR = false>
cudaError_t prepare_one() {
  return cudaFuncSetAttribute(tc_gemm_kernel<BN, SWAP, EPI, PAIR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              TileCfg<BN, SWAP, EPI, PAIR>::kSmem);
}

int g_num_sms = 0;
int g_max_pairs = 0;  // clusters of two 227 KB CTAs the device holds at once

// Launch as clusters of `cluster` CTAs, with programmatic dependent launch
// like launch_k.
template <typename... KArgs, typename... Args>
cudaError_t launch_clusters(void (*kernel)(KArgs...), int cluster, int clusters, size_t smem, cudaStream_t s,
                            Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cluster * clusters);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}
// Clusters of two CTAs (pairs of SMs).
template <typename... KArgs, typename... Args>
cudaError_t launch_pairs(void (*kernel)(KArgs...), int pairs, size_t smem, cudaStream_t s, Args... args) {
  return launch_clusters(kernel, 2, pairs, smem, s, args...);
}

// Output rows of one tile row (the stream-K tile): 128, or 256 for a pair.
int tile_rows(const TcGemm& t) { return t.pair ? 2 * BM : BM; }

// Stream-K units of a launch (CTAs, or CTA pairs): swapped -- tiles x splits;
// normal -- max_ctas (or one CTA per SM), halved for pairs; never more units
// than k-blocks.
int units_of(const TcGemm& t) {
  const int kb = (t.K + BK - 1) / BK;
  const long long tiles = (long long)((t.rows_a + tile_rows(t) - 1) / tile_rows(t)) * ((t.rows_b + t.bn - 1) / t.bn);
  long long want;
  if (t.swap) {
    int splits = t.splits < 1 ? 1 : t.splits;
    if (splits > kb) splits = kb;
    want = tiles * splits;
  } else {
    want = t.max_ctas > 0 ? t.max_ctas : g_num_sms;
    if (t.pair) {
      want /= 2;
      if (g_max_pairs > 0 && want > g_max_pairs) want = g_max_pairs;
    }
  }
  const long long W = tiles * kb;
  if (want > W) want = W;
  if (want < 1) want = 1;
  return (int)want;
}
int ctas_of(const TcGemm& t) { return units_of(t) * (t.pair ? 2 : 1); }

template <int BN, bool SWAP, int EPI, bool PAIR = false>
cudaError_t launch_one(const TcGemm& t, const EpiArgs& e, cudaStream_t s) {
  using C = TileCfg<BN, SWAP, EPI, PAIR>;
  GemmK g;
  g.rows_a = t.rows_a;
  g.rows_b = t.rows_b;
  g.K = t.K;
  g.z_a = t.z_a;
  g.z_b = t.z_b;
  g.tiles_a = (t.rows_a + tile_rows(t) - 1) / tile_rows(t);
  g.KB = (t.K + BK - 1) / BK;
  g.W = (long long)g.tiles_a * ((t.rows_b + BN - 1) / BN) * g.KB;
  g.G = units_of(t);
  g.ws = t.ws;
  g.tickets = t.tickets;
  g.status = t.status;
  g.csplit = (!PAIR && !SWAP && t.csplit && g.G % 2 == 0) ? 1 : 0;
  g.cred = 0;
  if (SWAP && !PAIR && t.cred > 1 && t.cred == t.splits) {
    // one cluster per tile, one equal k-range per CTA, the exchange areas (S
    // slices in, S - 1 out) fitting the operand ring
    const int S = t.cred;
    const long long tiles = (long long)g.tiles_a * ((t.rows_b + BN - 1) / BN);
    if (S > 8 || g.KB % S != 0 || BN % (4 * S) != 0 || g.G != tiles * S ||
        (size_t)C::kStages * C::kStageBytes < (size_t)(2 * S - 1) * BM * (BN / S) * 4)
      return cudaErrorInvalidValue;
    g.cred = S;
  }
  // unused output maps are passed as copies of the A map
  const CUtensorMap& mo = e.map_o ? *e.map_o : *t.map_a;
  const CUtensorMap& mo2 = e.map_o2 ? *e.map_o2 : *t.map_a;
  if constexpr (PAIR)
    return launch_pairs(tc_gemm_kernel<BN, SWAP, EPI, true>, g.G, C::kSmem, s, *t.map_a, *t.map_b, mo, mo2, g, e);
  else if (g.csplit)  // clusters of two CTAs: grid 2 x (G / 2)
    return launch_pairs(tc_gemm_kernel<BN, SWAP, EPI, false>, g.G / 2, C::kSmem, s, *t.map_a, *t.map_b, mo, mo2, g, e);
  else if (g.cred > 1)  // one cluster of g.cred CTAs per tile
    return launch_clusters(tc_gemm_kernel<BN, SWAP, EPI, false>, g.cred, (int)(g.G / g.cred), C::kSmem, s, *t.map_a,
                           *t.map_b, mo, mo2, g, e);
  else
    return launch_k(tc_gemm_kernel<BN, SWAP, EPI, false>, dim3(g.G), dim3(kThreads), C::kSmem, s, *t.map_a, *t.map_b,
                    mo, mo2, g, e);
}

template <int BN, bool PAIR = false>
cudaError_t launch_normal(const TcGemm& t, const EpiArgs& e, cudaStream_t s) {
  switch (e.kind) {
    case kEpiStoreF32:
    case kEpiGelu:
      if (!e.map_o) return cudaErrorInvalidValue;
      return launch_one<BN, false, kClassStore, PAIR>(t, e, s);
    case kEpiGateRes:
      if (!e.map_o) return cudaErrorInvalidValue;
      return launch_one<BN, false, kClassRes, PAIR>(t, e, s);
    case kEpiQkv:
      if (!e.map_o || !e.map_o2) return cudaErrorInvalidValue;
      return launch_one<BN, false, kClassQkv, PAIR>(t, e, s);
    default:
      if constexpr (PAIR)
        return cudaErrorInvalidValue;  // per-element epilogues run on single CTAs
      else
        return launch_one<BN, false, kClassScalar>(t, e, s);
  }
}

}  // namespace

size_t tc_gemm_ws_floats(const TcGemm& t) { return (size_t)ctas_of(t) * 2 * BM * t.bn; }

size_t tc_gemm_tickets(const TcGemm& t) {
  const int row_tiles = ((t.rows_a + tile_rows(t) - 1) / tile_rows(t)) * (t.pair ? 2 : 1);
  return (size_t)2 * row_tiles * ((t.rows_b + t.bn - 1) / t.bn);
}

namespace {
template <int BN, bool SWAP, int EPI>
int ring_partials() {
  using C = TileCfg<BN, SWAP, EPI>;
  return C::kStages * C::kStageBytes / (BM * BN * 4);
}
}  // namespace

int tc_gemm_ring_partials(int bn, bool swap, bool fused_norm) {
  if (swap && fused_norm) return bn == 32 ? ring_partials<32, true, kClassNormB>() : ring_partials<64, true, kClassNormB>();
  if (swap) {
    switch (bn) {
      case 32: return ring_partials<32, true, kClassScalar>();
      case 64: return ring_partials<64, true, kClassScalar>();
      case 128: return ring_partials<128, true, kClassScalar>();
      default: return ring_partials<256, true, kClassScalar>();
    }
  }
  return bn == 256 ? ring_partials<256, false, kClassQkv>() : ring_partials<128, false, kClassRes>();
}

cudaError_t prepare_tc_gemm() {
  cudaError_t e;
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
#define WAM_PREP(BN, SW, EP) \
  if ((e = prepare_one<BN, SW, EP>()) != cudaSuccess) return e;
  WAM_PREP(32, true, kClassScalar)
  WAM_PREP(64, true, kClassScalar)
  WAM_PREP(128, true, kClassScalar)
  WAM_PREP(256, true, kClassScalar)
  WAM_PREP(32, true, kClassNormB)
  WAM_PREP(64, true, kClassNormB)
  WAM_PREP(64, false, kClassScalar)
  WAM_PREP(64, false, kClassStore)
  WAM_PREP(64, false, kClassRes)
  WAM_PREP(64, false, kClassQkv)
  WAM_PREP(128, false, kClassScalar)
  WAM_PREP(128, false, kClassStore)
  WAM_PREP(128, false, kClassRes)
  WAM_PREP(128, false, kClassQkv)
  WAM_PREP(256, false, kClassScalar)
  WAM_PREP(256, false, kClassStore)
  WAM_PREP(256, false, kClassQkv)
  WAM_PREP(256, false, kClassRes)
  WAM_PREP(192, false, kClassScalar)
  WAM_PREP(192, false, kClassStore)
  WAM_PREP(192, false, kClassQkv)
  WAM_PREP(192, false, kClassRes)
#undef WAM_PREP
  if ((e = prepare_one<256, false, kClassStore, true>()) != cudaSuccess) return e;
  if ((e = prepare_one<256, false, kClassRes, true>()) != cudaSuccess) return e;
  if ((e = prepare_one<256, false, kClassQkv, true>()) != cudaSuccess) return e;
  {
    // how many pairs fit at once (SMs pair up within a GPC; some may be left over)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = TileCfg<256, false, kClassRes, true>::kSmem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, tc_gemm_kernel<256, false, kClassRes, true>, &cfg) != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = g_num_sms / 2;
    }
    g_max_pairs = n;
  }
  return cudaSuccess;
}

int tc_gemm_max_pairs() { return g_max_pairs; }

#ifdef WAM_GEMM_TIMELINE
extern "C" int wam_debug_gemm_timeline(unsigned long long* host, int n) {
  if (n > 1024) n = 1024;
  const int r = cudaMemcpyFromSymbol(host, g_gemm_tl, sizeof(unsigned long long) * 16 * n) == cudaSuccess ? g_max_pairs : -1;
  static unsigned long long zero[1024][16];
  cudaMemcpyToSymbol(g_gemm_tl, zero, sizeof zero);
  return r;
}
#endif

cudaError_t set_peer_wait_test(int extra, unsigned long long limit_ns) {
  cudaError_t e = cudaMemcpyToSymbol(g_peer_wait_extra, &extra, sizeof extra);
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_peer_wait_limit_ns, &limit_ns, sizeof limit_ns);
  return e;
}

cudaError_t launch_tc_gemm(const TcGemm& t, const EpiArgs& e, cudaStream_t s) {
  if (g_num_sms == 0) return cudaErrorNotReady;
  if (!t.ws || !t.tickets) return cudaErrorInvalidValue;
  // norm prologue: normal orientation, rows of at most 32 * 4 * kRowNormV values
  if (e.na_x && (t.swap || !e.na_h || !e.na_cnt || !e.na_scale || t.K % 4 || t.K > 32 * 4 * kRowNormV))
    return cudaErrorInvalidValue;
  if (e.nb_x) {  // fused norm of the token rows: swapped, one token tile, K <= kNormKMax
    if (!t.swap || t.rows_b > t.bn || t.K > kNormKMax || t.K % BK)
      return cudaErrorInvalidValue;
    switch (t.bn) {
      case 32: return launch_one<32, true, kClassNormB>(t, e, s);
      case 64: return launch_one<64, true, kClassNormB>(t, e, s);
    }
    return cudaErrorInvalidValue;
  }
  if (t.pair) {  // CTA pairs: normal orientation, 256-wide tiles
    if (t.swap || t.bn != 256 || t.rows_b % 32 != 0) return cudaErrorInvalidValue;
    return launch_normal<256, true>(t, e, s);
  }
  if (t.swap) {
    switch (t.bn) {
      case 32: return launch_one<32, true, kClassScalar>(t, e, s);
      case 64: return launch_one<64, true, kClassScalar>(t, e, s);
      case 128: return launch_one<128, true, kClassScalar>(t, e, s);
      case 256: return launch_one<256, true, kClassScalar>(t, e, s);
    }
  } else {
    // the normal orientation's epilogue writes whole 32-feature groups
    if (t.rows_b % 32 != 0) return cudaErrorInvalidValue;
    switch (t.bn) {
      case 64: return launch_normal<64>(t, e, s);
      case 128: return launch_normal<128>(t, e, s);
      case 192: return launch_normal<192>(t, e, s);
      case 256: return launch_normal<256>(t, e, s);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace wam
