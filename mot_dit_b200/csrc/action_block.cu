// Persistent action-expert block kernel for sm_100a: chunks of at most 32
// action tokens, bound by streaming the action weights and the block's K/V
// from HBM.
//
// One launch runs the action expert from one CEWP wait to the next:
// Attn^a_i, then R^a_i (out-projection + gate-residual, FFN up + GELU, FFN
// down + gate-residual), then P^a_{i+1} (norm + merged QKV + QK-norm + RoPE,
// writing the action rows of block i+1's K/V) -- or, after the last block, the
// final norm + output projection + Euler update.  The first launch of an Euler
// step runs the input projection and P^a_0.  Action block i's attention is
// thus the first thing of its launch, and the wait on the video expert's event
// e_i (RealtimeWAM summary page, 方法步骤详情: the action stream runs
// P^a_i -> wait(e_i) -> Attn^a_i -> R^a_i) stays between launches: no kernel
// waits on another launch.
//
// Dataflow inside a launch.  Every phase is a fixed set of work units -- 128
// weight rows x a fixed k-range (GEMMs), (sample, head, key split)
// (attention) -- chosen from the shapes and the SM count, never from the grid
// size; CTA c takes units c, c + G, ...  A unit waits only on what it reads:
// the out-projection's units on the attention splits of their heads, FFN-up
// and the next QKV on every tile of x_a, FFN-down on the FFN-up tiles of its
// k-range.  Completion is published through integer counters (one per tile /
// head), each released after a memory fence; every wait is bounded.  The grid
// is at most one CTA per SM and never larger than the SM count, so every unit
// waited on is resident.
//
// GEMMs are tcgen05.mma with the weight rows on the 128 TMEM lanes and the
// tokens as the N = 32 operand, fp32 accumulation in TMEM.  When a tile's
// k-range is split, every unit publishes its fp32 partial, and once all have,
// unit s sums token slice s of the tile over the splits in split order and
// applies the epilogue: the result depends neither on the grid size nor on
// timing, so every schedule is bitwise equal.  Epilogues that update x_a also
// publish the per-tile row sums of squares, so the RMSNorm of the next phase
// reads only its own columns of x_a.
//
// Warp roles (192 threads):
//   warp 0     weight producer: one thread streams every weight k-block of the
//              launch (all phases, in order) through a TMA ring; weights do not
//              depend on the dataflow, so later phases' tiles are in flight
//              while earlier ones wait.
//   warp 1     TMEM owner and MMA issuer (one thread).
//   warps 2-5  compute: dependency waits, the B operand of each phase (TMA
//              loads of the activations, the RMSNorm / AdaLN modulation of x_a,
//              or the attention output combined from its splits, written
//              straight into the swizzled K-major layout), the attention
//              softmax, the split reductions and the epilogues.
//
// Attention of action block i over the joint keys [K^v_i; K^a_i] (rows
// [0, L_v + L_a) of the block's cache; summary page, 前置知识
// "Mixture-of-Transformers"): units are (sample, head, key split).  S = Q K^T
// is one M = 128 MMA over the split's keys (the <= 32 queries padded with
// zero rows by the TMA fill); the thread of query q reads its scores from
// TMEM and writes P (bf16) into the K-major operand tiles over Q and K; O =
// P V accumulates in TMEM with V as the MN-major operand.  Each unit
// publishes (row maximum, row sum, O); the out-projection combines the splits
// of its heads in split order while it builds its operand.
//
// Every wait is bounded by %globaltimer (common.cuh): a wait that gives up
// sets a bit in the status word and the CTA winds down -- it drains its TMA
// copies and its MMAs before releasing TMEM; no trap, no endless spin.
#include "common.cuh"
#include "kernels.h"

namespace wam {
namespace {

constexpr int kThr = 192;
constexpr int BM = 128, BK = 64, BN = 32;
constexpr int kStages = 6;
constexpr int kTileA = BM * BK * 2;             // 16 KB weight k-block
constexpr int kBBlk = BN * 128;                 // 4 KB activation k-block (32 tokens x 64)
constexpr int kRegion = 80 * 1024;              // B k-blocks, or V | Q | K of one attention unit
constexpr int kRegionSlots = kRegion / kBBlk;   // 20 B k-blocks
constexpr int kStgLd = BM + 1;
constexpr int kStg = BN * kStgLd * 4;           // [32 tokens][129] fp32 staging
constexpr int kBarBytes = 1024;                 // mbarriers, flags, per-warp row sums
constexpr int kSmem = kStages * kTileA + kRegion + kStg + kBarBytes;
constexpr int kTmemCols = 512;                  // acc[2] at 0 / 32, S at 64.., O at 320..383
constexpr int kTmemS = 64, kTmemO = 320;
constexpr int kMaxTiles = kActionBlockMaxTiles;
constexpr int kPh = kActionBlockPhases;
constexpr int kAttnPart = BN * 64 + 2 * BN;     // one attention partial: O [32][64], m [32], l [32]
constexpr int kMaps = kActionBlockMaps;
constexpr int kMaxSplits = 16;                  // attention key splits combined in one pass
// Counter layout (ints): [phase][published, done][tile], then [phase] operand
// built, then the exit ticket.
constexpr int kCntPub = 0, kCntDone = 1;
constexpr int kCntBuilt = kPh * 2 * kMaxTiles;
constexpr int kCntExit = kCntBuilt + kPh;
constexpr int kCntInts = kCntExit + 1;

__device__ __forceinline__ int* cnt_tile(int* cnt, int phase, int which, int t) {
  return cnt + (phase * 2 + which) * kMaxTiles + t;
}

__device__ __forceinline__ void bar_compute() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ void arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void fence_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// Shared-memory descriptor of an MN-major bf16 operand stored as 128-byte rows
// (64 elements along N) with the 128-byte swizzle, consecutive K rows 128 B
// apart, 8-row groups 1024 B apart: a TMA SWIZZLE_128B tile of [K][64].
__device__ __forceinline__ uint64_t desc_mn128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>(1) << 16;
  d |= static_cast<uint64_t>(1024 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// 32 lanes x 64 consecutive 32-bit TMEM columns.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
  float (&lo)[32] = *reinterpret_cast<float(*)[32]>(&v[0]);
  float (&hi)[32] = *reinterpret_cast<float(*)[32]>(&v[32]);
  tmem_ld32(taddr, lo);
  tmem_ld32(taddr + 32, hi);
}

// 2^x on the special-function unit (relative error far below bf16 rounding).
__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Bounded spin until *p >= target (p written by other CTAs of this grid, all
// resident).  False -- status bit and abort flag set -- when the limit passes.
__device__ __forceinline__ bool wait_geq(const int* p, int target, unsigned* status, volatile int* abort_flag) {
  const volatile int* vp = p;
  if (*vp >= target) return true;
  const unsigned long long t0 = globaltimer();
  while (*vp < target) {
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitLimitNs) {
      atomicOr(status, kStatusTimeoutPeer);
      *abort_flag = 1;
      return false;
    }
  }
  return true;
}

// Releases this CTA's writes (all 128 compute threads') and bumps a counter
// other CTAs wait on.  Called by every compute thread.
__device__ __forceinline__ void publish(int* counter) {
  bar_compute();
  if (threadIdx.x == 64) {
    __threadfence();
    atomicAdd(counter, 1);
  }
}

// Diagnostic build (-DWAM_AB_PHASES): thread 64 of every CTA stamps
// %globaltimer at the phase boundaries of the latest launch into
// g_ab_phase[cta][k]; the normal build compiles none of it.
#ifdef WAM_AB_PHASES
__device__ unsigned long long g_ab_phase[160][32];
#define AB_STAMP(k)                                                        \
  do {                                                                     \
    if (threadIdx.x == 64 && blockIdx.x < 160 && (k) < 32) g_ab_phase[blockIdx.x][(k)] = globaltimer(); \
  } while (0)
#else
#define AB_STAMP(k) \
  do {              \
  } while (0)
#endif

using GPh = ActionGemmPhase;
using ActArgs = ActionBlockArgs;
using ActMaps = ActionBlockMaps;

__device__ __forceinline__ int units_of(const GPh& p) { return ((p.n_out + BM - 1) / BM) * p.ks; }
__device__ __forceinline__ void krange(const GPh& p, int s, int& kb0, int& kb1) {
  const int KB = p.K / BK;
  kb0 = s * KB / p.ks;
  kb1 = (s + 1) * KB / p.ks;
}
// k-blocks of the phase that CTA `cta` of G reads, as a bit mask (K <= 4096).
__device__ __host__ __forceinline__ unsigned long long kb_mask_of(int n_out, int K, int ks, int cta, int G) {
  unsigned long long m = 0;
  const int U = ((n_out + BM - 1) / BM) * ks, KB = K / BK;
  for (int u = cta; u < U; u += G) {
    const int s = u % ks;
    for (int kb = s * KB / ks; kb < (s + 1) * KB / ks; ++kb) m |= 1ull << kb;
  }
  return m;
}
__device__ __forceinline__ unsigned long long kb_mask(const GPh& p, int cta, int G) {
  return kb_mask_of(p.n_out, p.K, p.ks, cta, G);
}
__device__ __forceinline__ int slot_of(unsigned long long mask, int kb) {
  return __popcll(mask & ((1ull << kb) - 1ull));
}

// Per-head QK-RMSNorm (gain g[64]) then rotate-half RoPE (cos / sin rows of
// the token's position).
__device__ __forceinline__ void qk_norm_rope64(float (&x)[64], const float* g, const float* cs, const float* sn) {
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < 64; ++j) ss += x[j] * x[j];
  const float r = rsqrtf(ss * (1.0f / 64.0f) + 1e-6f);
#pragma unroll
  for (int j = 0; j < 64; ++j) x[j] *= r * __ldg(g + j);
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float c = __ldg(cs + j), s = __ldg(sn + j);
    const float x1 = x[j], x2 = x[j + 32];
    x[j] = x1 * c - x2 * s;
    x[j + 32] = x1 * s + x2 * c;
  }
}

__device__ __forceinline__ void store64_bf16(__nv_bfloat16* dst, const float (&x)[64]) {
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

// Row sums of squares of new x_a values over the 128 features of a tile: each
// compute thread holds feature f's values of tokens m0 .. m0 + nm - 1; the sum
// runs in a fixed order (warp tree, then the four warps in order) and lands in
// ss_tile[m0 + j].  Every compute thread calls it.
__device__ __forceinline__ void tile_row_ss(const float (&xn)[32], int nm, float* red4, float* ss_tile, int m0) {
  const int lane = threadIdx.x & 31, w = (threadIdx.x >> 5) - 2;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    if (j >= nm) break;
    float v = xn[j] * xn[j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red4[w * 32 + j] = v;
  }
  bar_compute();
  const int te = threadIdx.x - 64;
  if (te < nm) ss_tile[m0 + te] = ((red4[te] + red4[32 + te]) + red4[64 + te]) + red4[96 + te];
  bar_compute();
}

// Epilogue of a slice of one tile, run by all 128 compute threads: the thread
// owns feature n = tile * 128 + f, v[j] = the sum (bias not added) for token
// m0 + j (j < nm) and xo[j] the old value the epilogue updates (x_a, the
// action state).  QKV items go through the staging buffer; every thread
// reaches the barriers.
__device__ __forceinline__ void epilogue(const ActArgs& a, const GPh& p, int tile, int f, int m0, int nm,
                                         const float (&v)[32], const float (&xo)[32], float* stg, float* red4) {
  const int n = tile * BM + f;
  const bool n_ok = n < p.n_out;
  const float b = n_ok ? __ldg(p.bias + n) : 0.f;
  if (p.epi == kEpiQkv) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < nm) stg[j * kStgLd + f] = v[j] + b;
    bar_compute();
    const int te = threadIdx.x - 64;
    for (int it = te; it < nm * 2; it += 128) {  // items: (token j, head hh of the tile's two)
      const int j = it % nm, hh = it / nm;
      const int n0 = tile * BM + hh * 64;
      if (n0 >= p.n_out) continue;
      const int m = m0 + j;
      const int bidx = m / a.La, l = m - bidx * a.La;
      float x[64];
#pragma unroll
      for (int k = 0; k < 64; ++k) x[k] = stg[j * kStgLd + hh * 64 + k];
      const int section = n0 / a.A, head = (n0 % a.A) / 64;
      const int pos = a.cache_off + l;
      if (section < 2)
        qk_norm_rope64(x, (section == 0 ? p.gq : p.gk) + head * 64, a.rope_cos + pos * 32, a.rope_sin + pos * 32);
      __nv_bfloat16* dst;
      if (section == 0)
        dst = p.q_out + ((size_t)(bidx * a.H + head) * a.La + l) * 64;
      else
        dst = (section == 1 ? p.k_cache : p.v_cache) +
              ((size_t)(bidx * a.H + head) * a.cache_len + a.cache_off + l) * 64;
      store64_bf16(dst, x);
    }
    bar_compute();  // the staging is free again
    return;
  }
  if (p.epi == kEpiGateRes || p.epi == kEpiStoreF32) {
    // new x_a values, stored, and their row sums of squares per tile
    const float g = (p.epi == kEpiGateRes && n_ok) ? __ldg(p.gate + n) : 0.f;
    float xn[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) xn[j] = n_ok ? (p.epi == kEpiGateRes ? xo[j] + g * (v[j] + b) : v[j] + b) : 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < nm && n_ok) p.out_f32[(size_t)(m0 + j) * p.ld_out + n] = xn[j];
    if (p.ss_out >= 0)
      tile_row_ss(xn, nm, red4, a.ss + ((size_t)p.ss_out * (a.da / BM) + tile) * a.Ma, m0);
    return;
  }
  if (!n_ok) return;
  switch (p.epi) {
    case kEpiGelu:
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (j >= nm) break;
        p.out_act[(size_t)(m0 + j) * p.ld_out + n] = __float2bfloat16_rn(gelu_tanh(v[j] + b));
      }
      break;
    case kEpiEuler: {
      const float dt = a.aio->sched[p.step] - a.aio->sched[p.step + 1];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (j >= nm) break;
        const float an = xo[j] - dt * (v[j] + b);
        p.out_f32[(size_t)(m0 + j) * p.ld_out + n] = an;
        if (p.a_next) p.a_next[(size_t)(m0 + j) * p.a_next_ld + n] = __float2bfloat16_rn(an);
      }
      break;
    }
    default:
      break;
  }
}

// Old values the epilogue updates in place (x_a for the gate-residual, the
// action state for the Euler update), all loads in flight together.
__device__ __forceinline__ void load_old(const GPh& p, int n, int m0, int nm, float (&xo)[32]) {
  const bool rd = (p.epi == kEpiGateRes || p.epi == kEpiEuler) && n < p.n_out;
#pragma unroll
  for (int j = 0; j < 32; ++j) xo[j] = (rd && j < nm) ? __ldcg(p.out_f32 + (size_t)(m0 + j) * p.ld_out + n) : 0.f;
}

__global__ void __launch_bounds__(kThr, 1)
    action_block_kernel(const __grid_constant__ ActMaps maps, const __grid_constant__ ActArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023) {
    if (threadIdx.x == 0) atomicOr(a.status, kStatusTimeoutDrain);
    return;
  }
  uint8_t* ring = smem_raw;                   // [kStages][16 KB] weight k-blocks
  uint8_t* region = ring + kStages * kTileA;  // B k-blocks, or V | Q | K (P over Q | K)
  float* stg = reinterpret_cast<float*>(region + kRegion);
  uint64_t* bars = reinterpret_cast<uint64_t*>(region + kRegion + kStg);
  uint64_t* full = bars;             // [kStages] weight k-block landed
  uint64_t* empty = full + kStages;  // [kStages] weight k-block read by the MMAs
  uint64_t* accf = empty + kStages;  // [2] accumulator ready
  uint64_t* acce = accf + 2;         // [2] accumulator drained (one arrival per compute warp)
  uint64_t* bready = acce + 2;       // B operand of a GEMM phase in place
  uint64_t* kvfull = bready + 1;     // V, Q, K of an attention unit landed
  uint64_t* sfull = kvfull + 1;      // S computed
  uint64_t* pfull = sfull + 1;       // P written (32 softmax threads)
  uint64_t* ofull = pfull + 1;       // O computed (P and V read)
  uint64_t* mdone = ofull + 1;       // every MMA of this CTA complete (teardown)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mdone + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = abort_flag + 1;
  float* red4 = reinterpret_cast<float*>(bars + 32);  // [4][32] per-warp row sums

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int n_attn_units = a.has_attn ? a.B * a.H * a.at.splits : 0;
  const int kps = a.at.keys;                                           // keys per attention split
  const uint32_t v_off = 0, q_off = kps * 128, k_off = q_off + 16384;  // V | Q | K in the region

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], 4);
    }
    mbar_init(bready, 1);
    mbar_init(kvfull, 1);
    mbar_init(sfull, 1);
    mbar_init(pfull, 32);
    mbar_init(ofull, 1);
    mbar_init(mdone, 1);
    *abort_flag = 0;
    *last_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < kMaps; ++i) prefetch_tensormap(&maps.m[i]);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------ weight producer
    // (weights never change during a chunk: no wait for the previous kernel)
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int pi = 0; pi < a.n_gemm && ok; ++pi) {
        const GPh& p = a.g[pi];
        const int U = units_of(p);
        for (int u = cta; u < U && ok; u += G) {
          const int t = u / p.ks;
          int kb0, kb1;
          krange(p, u % p.ks, kb0, kb1);
          for (int kb = kb0; kb < kb1; ++kb) {
            const int s = it % kStages;
            if (it >= kStages &&
                !mbar_wait(&empty[s], ((it / kStages) - 1) & 1, a.status, kStatusTimeoutTmaEmpty, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full[s], kTileA);
            tma_load_3d(ring + s * kTileA, &maps.m[p.map_w], &full[s], kb * BK, t * BM, p.z);
            ++it;
          }
        }
      }
      // never leave copies into this CTA's shared memory in flight
      for (int i = max(0, it - kStages); i < it; ++i)
        mbar_wait(&full[i % kStages], (i / kStages) & 1, a.status, kStatusTimeoutDrain, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      bool issued = false;
      int ua = 0;
      const uint32_t r0 = smem_u32(region);
      for (int u = cta; u < n_attn_units && ok; u += G, ++ua) {
        if (!mbar_wait(kvfull, ua & 1, a.status, kStatusTimeoutTmaFull, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t idesc_s = idesc_bf16_f32(128, kps);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 64) | (1u << 16);  // B (V) MN-major
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc_mma_bf16(tmem + kTmemS, smem_desc_k128(r0 + q_off + k * 32), smem_desc_k128(r0 + k_off + k * 32),
                      idesc_s, k > 0 ? 1u : 0u);
        tc_commit(sfull);
        issued = true;
        if (!mbar_wait(pfull, ua & 1, a.status, kStatusTimeoutAccum, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // P: kps / 64 K-major tiles [128 rows][128 B], 16 KB apart, from Q's offset
        for (int kk = 0; kk < kps / 16; ++kk)
          tc_mma_bf16(tmem + kTmemO, smem_desc_k128(r0 + q_off + (kk >> 2) * 16384 + (kk & 3) * 32),
                      desc_mn128(r0 + v_off + kk * 16 * 128), idesc_pv, kk > 0 ? 1u : 0u);
        tc_commit(ofull);
      }
      int it = 0, lt = 0;
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN);
      for (int pi = 0; pi < a.n_gemm && ok; ++pi) {
        const GPh& p = a.g[pi];
        if (!mbar_wait(bready, pi & 1, a.status, kStatusTimeoutTmaFull, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const unsigned long long mask = kb_mask(p, cta, G);
        const int U = units_of(p);
        for (int u = cta; u < U && ok; u += G, ++lt) {
          const int buf = lt & 1;
          if (lt >= 2 && !mbar_wait(&acce[buf], ((lt >> 1) - 1) & 1, a.status, kStatusTimeoutAccum, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          int kb0, kb1;
          krange(p, u % p.ks, kb0, kb1);
          for (int kb = kb0; kb < kb1; ++kb, ++it) {
            const int s = it % kStages;
            if (!mbar_wait(&full[s], (it / kStages) & 1, a.status, kStatusTimeoutTmaFull, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a0 = smem_u32(ring + s * kTileA);
            const uint32_t b0 = r0 + slot_of(mask, kb) * kBBlk;
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              tc_mma_bf16(tmem + buf * BN, smem_desc_k128(a0 + k * 32), smem_desc_k128(b0 + k * 32), idesc,
                          (kb > kb0 || k > 0) ? 1u : 0u);
            tc_commit(&empty[s]);
            issued = true;
          }
          if (!ok) break;
          tc_commit(&accf[buf]);
        }
      }
      // every MMA this thread issued has completed before TMEM is released
      if (issued) {
        tc_commit(mdone);
        mbar_wait(mdone, 0, a.status, kStatusTimeoutDrain, nullptr);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ compute warps
    AB_STAMP(0);
    pdl_wait();  // activations and the cache belong to earlier kernels until they finish
    AB_STAMP(1);
    const int te = threadIdx.x - 64;
    const int quad = warp & 3;  // TMEM lane quarter this warp may read
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const int row = quad * 32 + lane;  // TMEM lane of this thread = weight row within a tile
    bool ok = true;
    int kv_issued = 0;         // attention loads issued (phases of kvfull)
    int bready_last = -1;      // last GEMM phase whose bready this CTA armed
    bool bready_last_tma = false;

    // ---------------- attention units of the block: publish (m, l, O) per split
    if (n_attn_units > 0) {
      const float sl2e = 1.4426950408889634f * 0.125f;  // log2(e) / sqrt(64)
      int ua = 0;
      for (int u = cta; u < n_attn_units; u += G, ++ua) {
        const int bh = u / a.at.splits, sp = u % a.at.splits;
        if (te == 0) {
          // the previous unit's PV has read the region (P over Q | K, and V)
          if (ua > 0 && !mbar_wait(ofull, (ua - 1) & 1, a.status, kStatusTimeoutAccum, abort_flag)) {
            *abort_flag = 1;
          } else {
            fence_async_global();
            fence_async_smem();
            mbar_arrive_expect_tx(kvfull, 16384 + 2 * kps * 128);
            tma_load_3d(region + v_off, &maps.m[10], kvfull, 0, sp * kps, a.at.zv0 + bh);
            tma_load_3d(region + q_off, &maps.m[9], kvfull, 0, 0, bh);
            tma_load_3d(region + k_off, &maps.m[10], kvfull, 0, sp * kps, a.at.zk0 + bh);
            ++kv_issued;
          }
        }
        bar_compute();
        if (*abort_flag) {
          ok = false;
          break;
        }
        if (quad == 0) {
          // query `lane` (TMEM lane `lane`) over this unit's keys
          const int nvalid = min(kps, a.Lk - sp * kps);
          const uint32_t t_s = tmem + kTmemS, t_o = tmem + kTmemO;
          bool got = mbar_wait(sfull, ua & 1, a.status, kStatusTimeoutAccum, abort_flag);
          got = __all_sync(0xffffffffu, got) != 0;
          float mref = -INFINITY, lsum = 0.f;
          if (got) {
            tc_fence_after();
            float v[64];
            float mx = -INFINITY;
            for (int c0 = 0; c0 < kps; c0 += 64) {
              tmem_ld64(t_s + c0, v);
#pragma unroll
              for (int i = 0; i < 64; ++i)
                if (c0 + i < nvalid) mx = fmaxf(mx, v[i]);
            }
            mref = mx * sl2e;
            const int swz = lane & 7;
            for (int c0 = 0; c0 < kps; c0 += 64) {
              tmem_ld64(t_s + c0, v);
#pragma unroll
              for (int i = 0; i < 64; ++i) {
                const float pv = (c0 + i < nvalid) ? ex2f(fmaf(v[i], sl2e, -mref)) : 0.f;
                v[i] = pv;
                lsum += pv;
              }
              uint8_t* prow = region + q_off + (c0 / 64) * 16384 + lane * 128;
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                uint4 w;
                w.x = pack_bf16(v[8 * q + 0], v[8 * q + 1]);
                w.y = pack_bf16(v[8 * q + 2], v[8 * q + 3]);
                w.z = pack_bf16(v[8 * q + 4], v[8 * q + 5]);
                w.w = pack_bf16(v[8 * q + 6], v[8 * q + 7]);
                *reinterpret_cast<uint4*>(prow + ((q ^ swz) << 4)) = w;
              }
            }
            tc_fence_before();
            fence_async_smem();  // P (generic stores) -> tensor-core reads
            arrive(pfull);
            got = mbar_wait(ofull, ua & 1, a.status, kStatusTimeoutAccum, abort_flag);
            got = __all_sync(0xffffffffu, got) != 0;
          }
          if (got) {
            tc_fence_after();
            float o[64];
            tmem_ld64(t_o, o);
            if (lane < a.La) {
              float* part = a.ws_attn + (size_t)u * kAttnPart;
#pragma unroll
              for (int j = 0; j < 16; ++j)
                __stcg(reinterpret_cast<float4*>(part + lane * 64) + j,
                       make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]));
              __stcg(part + BN * 64 + lane, mref);
              __stcg(part + BN * 64 + BN + lane, lsum);
            }
          } else {
            *abort_flag = 1;
          }
        }
        publish(a.cnt_attn + bh);
        bar_compute();
        if (*abort_flag) {
          ok = false;
          break;
        }
      }
    }
    AB_STAMP(2);

    // ---------------- GEMM phases
    int lt = 0;
    for (int pi = 0; pi < a.n_gemm && ok; ++pi) {
      const GPh& p = a.g[pi];
      const unsigned long long mask = kb_mask(p, cta, G);
      const int nslots = __popcll(mask);
      if (nslots > kRegionSlots) {  // the host sizes the grid so that this never happens
        if (te == 0) {
          atomicOr(a.status, kStatusTimeoutTmaFull);
          *abort_flag = 1;
        }
        ok = false;
        break;
      }
      // wait for what this CTA's units read (nothing when it has none)
      if (te == 0 && mask) {
        const int pp = pi - 1;
        if (p.dep == kDepAll && pp >= 0) {
          const GPh& q = a.g[pp];
          const int tq = (q.n_out + BM - 1) / BM;
          for (int t2 = 0; t2 < tq && !*abort_flag; ++t2)
            wait_geq(cnt_tile(a.cnt, pp, kCntDone, t2), q.ks, a.status, abort_flag);
        } else if (p.dep == kDepKRange && pp >= 0) {
          const GPh& q = a.g[pp];
          for (int kb = 0; kb < p.K / BK && !*abort_flag; ++kb)
            if (mask >> kb & 1ull) wait_geq(cnt_tile(a.cnt, pp, kCntDone, kb * BK / BM), q.ks, a.status, abort_flag);
        } else if (p.dep == kDepHeads) {
          for (int kb = 0; kb < p.K / BK && !*abort_flag; ++kb)
            if (mask >> kb & 1ull)
              for (int b = 0; b < a.B && !*abort_flag; ++b)
                wait_geq(a.cnt_attn + b * a.H + kb, a.at.splits, a.status, abort_flag);
        }
        __threadfence();
      }
      bar_compute();
      if (*abort_flag) {
        ok = false;
        break;
      }
      AB_STAMP(4 + 4 * pi);
      // B operand of the phase
      if (p.bsrc == kBTma) {
        if (te == 0) {
          fence_async_global();
          fence_async_smem();
          mbar_arrive_expect_tx(bready, nslots * kBBlk);
          for (int kb = 0; kb < p.K / BK; ++kb)
            if (mask >> kb & 1ull)
              tma_load_3d(region + slot_of(mask, kb) * kBBlk, &maps.m[p.map_b], bready, kb * BK, 0, 0);
          bready_last = pi;
          bready_last_tma = true;
        }
      } else {
        const int r = te >> 2, part = te & 3;  // token r, columns [16 part, 16 part + 16) of each k-block
        const bool valid = r < a.Ma;
        if (p.bsrc == kBNorm) {
          // rms(x_a) (gain | 1 + scale) + shift; 1/rms from the row sums of
          // squares the producing tiles published (fixed order over tiles)
          float rr = 0.f;
          if (valid && mask) {
            const float* ssb = a.ss + (size_t)p.ss_in * (a.da / BM) * a.Ma + r;
            float sum = 0.f;
            for (int t2 = 0; t2 < a.da / BM; ++t2) sum += __ldcg(ssb + (size_t)t2 * a.Ma);
            rr = 1.0f / sqrtf(sum / (float)a.da + 1e-6f);
          }
          const float4* xr = reinterpret_cast<const float4*>(a.x_a + (size_t)(valid ? r : 0) * a.da);
          for (int kb = 0; kb < p.K / BK; ++kb) {
            if (!(mask >> kb & 1ull)) continue;
            const int c0 = kb * BK + part * 16;
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              float4 mul, add = make_float4(0.f, 0.f, 0.f, 0.f);
              if (p.ngain) {
                mul = __ldg(reinterpret_cast<const float4*>(p.ngain + c0) + i);
              } else {
                mul = __ldg(reinterpret_cast<const float4*>(p.nscale + c0) + i);
                mul.x += 1.f;
                mul.y += 1.f;
                mul.z += 1.f;
                mul.w += 1.f;
              }
              if (p.nshift) add = __ldg(reinterpret_cast<const float4*>(p.nshift + c0) + i);
              const float4 x4 = valid ? __ldcg(xr + c0 / 4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
              w[2 * i] = valid ? pack_bf16(x4.x * rr * mul.x + add.x, x4.y * rr * mul.y + add.y) : 0u;
              w[2 * i + 1] = valid ? pack_bf16(x4.z * rr * mul.z + add.z, x4.w * rr * mul.w + add.w) : 0u;
            }
            uint8_t* rowp = region + slot_of(mask, kb) * kBBlk + r * 128;
            const int q = part * 2;
            *reinterpret_cast<uint4*>(rowp + ((q ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
            *reinterpret_cast<uint4*>(rowp + (((q + 1) ^ (r & 7)) << 4)) = make_uint4(w[4], w[5], w[6], w[7]);
          }
        } else {
          // attention output: k-block kb = head kb; its splits combined in
          // split order with log-sum-exp weights, rounded to bf16
          const int S2 = a.at.splits;
          const int bidx = valid ? r / a.La : 0, q = valid ? r - bidx * a.La : 0;
          for (int kb = 0; kb < p.K / BK; ++kb) {
            if (!(mask >> kb & 1ull)) continue;
            const float* base = a.ws_attn + (size_t)(bidx * a.H + kb) * S2 * kAttnPart;
            float ms[kMaxSplits], ls[kMaxSplits];
#pragma unroll
            for (int s2 = 0; s2 < kMaxSplits; ++s2) {
              const bool on = valid && s2 < S2;
              ms[s2] = on ? __ldcg(base + (size_t)s2 * kAttnPart + BN * 64 + q) : -INFINITY;
              ls[s2] = on ? __ldcg(base + (size_t)s2 * kAttnPart + BN * 64 + BN + q) : 0.f;
            }
            float M = -INFINITY;
#pragma unroll
            for (int s2 = 0; s2 < kMaxSplits; ++s2) M = fmaxf(M, ms[s2]);
            float den = 0.f;
#pragma unroll
            for (int s2 = 0; s2 < kMaxSplits; ++s2) {
              ms[s2] = (valid && s2 < S2) ? ex2f(ms[s2] - M) : 0.f;  // the split's weight
              den += ms[s2] * ls[s2];
            }
            const float inv = valid ? 1.0f / den : 0.f;
            float acc[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) acc[i] = 0.f;
#pragma unroll
            for (int s2 = 0; s2 < kMaxSplits; ++s2) {
              if (s2 >= S2) break;
              const float4* po = reinterpret_cast<const float4*>(base + (size_t)s2 * kAttnPart + q * 64 + part * 16);
              float4 o4[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) o4[i] = valid ? __ldcg(po + i) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                acc[4 * i] += ms[s2] * o4[i].x;
                acc[4 * i + 1] += ms[s2] * o4[i].y;
                acc[4 * i + 2] += ms[s2] * o4[i].z;
                acc[4 * i + 3] += ms[s2] * o4[i].w;
              }
            }
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) w[i] = valid ? pack_bf16(acc[2 * i] * inv, acc[2 * i + 1] * inv) : 0u;
            uint8_t* rowp = region + slot_of(mask, kb) * kBBlk + r * 128;
            const int qc = part * 2;
            *reinterpret_cast<uint4*>(rowp + ((qc ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
            *reinterpret_cast<uint4*>(rowp + (((qc + 1) ^ (r & 7)) << 4)) = make_uint4(w[4], w[5], w[6], w[7]);
          }
        }
        fence_async_smem();
        bar_compute();
        if (te == 0) {
          arrive(bready);
          bready_last = pi;
          bready_last_tma = false;
        }
      }
      // this CTA has read what its operand needed (x_a, for a norm): later
      // writers of x_a in the launch wait until every CTA has
      if (te == 0) atomicAdd(a.cnt + kCntBuilt + pi, 1);
      AB_STAMP(5 + 4 * pi);
      // the units: accumulate, then finish (whole k-range) or publish (k-split)
      const int U = units_of(p);
      float* wsp = a.ws + (size_t)(pi & 1) * a.ws_half;
      for (int u = cta; u < U; u += G, ++lt) {
        const int buf = lt & 1;
        const int t = u / p.ks;
        float xo[32];
        if (p.ks == 1) load_old(p, t * BM + row, 0, a.Ma, xo);  // (in flight during the wait)
        const bool got = mbar_wait(&accf[buf], (lt >> 1) & 1, a.status, kStatusTimeoutAccum, abort_flag);
        if (!__all_sync(0xffffffffu, got)) *abort_flag = 1;
        bar_compute();
        if (*abort_flag) {
          ok = false;
          break;
        }
        tc_fence_after();
        float v[32];
        tmem_ld32(t_lane + buf * BN, v);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive(&acce[buf]);
        if (p.ks == 1) {
          if (p.war_phase >= 0 && te == 0) wait_geq(a.cnt + kCntBuilt + p.war_phase, G, a.status, abort_flag);
          bar_compute();
          epilogue(a, p, t, row, 0, a.Ma, v, xo, stg, red4);
          publish(cnt_tile(a.cnt, pi, kCntDone, t));
        } else {
          float* part = wsp + (size_t)u * (BN * BM);
#pragma unroll
          for (int j = 0; j < 32; ++j) __stcg(part + j * BM + row, v[j]);
          publish(cnt_tile(a.cnt, pi, kCntPub, t));
        }
      }
      AB_STAMP(6 + 4 * pi);
      if (!ok || p.ks == 1) continue;
      // split reduction: unit (t, s) sums token slice s of tile t over the splits, in order
      const int per = (a.Ma + p.ks - 1) / p.ks;
      for (int u = cta; u < U; u += G) {
        const int t = u / p.ks, s = u % p.ks;
        const int m0 = s * per, nm = max(0, min(per, a.Ma - m0));
        float xo[32];
        load_old(p, t * BM + te, m0, nm, xo);  // (in flight during the waits)
        if (te == 0) {
          wait_geq(cnt_tile(a.cnt, pi, kCntPub, t), p.ks, a.status, abort_flag);
          if (p.war_phase >= 0) wait_geq(a.cnt + kCntBuilt + p.war_phase, G, a.status, abort_flag);
          __threadfence();
        }
        bar_compute();
        if (*abort_flag) {
          ok = false;
          break;
        }
        // every split's slice [nm tokens][128 features] into the region (free:
        // this CTA's MMAs of the phase are complete), all copies in flight at
        // once, then the sums in split order from shared memory
        float* red = reinterpret_cast<float*>(region);  // [ks][nm][128]
        const int n16 = p.ks * nm * (BM / 4);
        for (int i = te; i < n16; i += 128) {
          const int s2 = i / (nm * (BM / 4)), rem = i - s2 * (nm * (BM / 4));
          cp_async16(smem_u32(red + 4 * i), wsp + ((size_t)(t * p.ks + s2) * BN + m0) * BM + 4 * rem, true);
        }
        cp_async_commit();
        cp_async_wait<0>();
        bar_compute();
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          float acc = 0.f;
          if (j < nm)
            for (int s2 = 0; s2 < p.ks; ++s2) acc += red[(s2 * nm + j) * BM + te];
          v[j] = acc;
        }
        bar_compute();  // the region is read before anything else may reuse it
        epilogue(a, p, t, te, m0, nm, v, xo, stg, red4);
        publish(cnt_tile(a.cnt, pi, kCntDone, t));
      }
      AB_STAMP(7 + 4 * pi);
    }
    // ---------------- exit: the last CTA out leaves every counter at zero
    bar_compute();
    if (te == 0) {
      __threadfence();
      *last_flag = atomicAdd(a.cnt + kCntExit, 1) == G - 1 ? 1 : 0;
    }
    bar_compute();
    if (*last_flag) {
      __threadfence();
      for (int i = te; i < kCntExit; i += 128) a.cnt[i] = 0;
      for (int i = te; i < a.B * a.H; i += 128) a.cnt_attn[i] = 0;
      bar_compute();
      if (te == 0) {
        a.cnt[kCntExit] = 0;
        __threadfence();
      }
    }
    // No TMA copy this thread issued may still be landing at exit.  (On the
    // normal path the MMA thread has waited for all of them; after an abort
    // only the last one armed can be outstanding: every earlier one was waited
    // for before the next was issued.)
    if (te == 0) {
      if (kv_issued > 0) mbar_wait(kvfull, (kv_issued - 1) & 1, a.status, kStatusTimeoutDrain, nullptr);
      if (bready_last >= 0 && bready_last_tma) mbar_wait(bready, bready_last & 1, a.status, kStatusTimeoutDrain, nullptr);
    }
  }

  // ------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

// ---------------------------------------------------------------- host side
int action_block_ks(int n_out, int K, int nsm) {
  const int tiles = (n_out + BM - 1) / BM, KB = K / BK;
  int ks = nsm / tiles;
  if (ks > KB) ks = KB;
  if (ks < 1) ks = 1;
  return ks;
}

bool action_block_fits(int n_out, int K, int ks, int G) {
  if (K % BK || K / BK > 64 || (n_out + BM - 1) / BM > kMaxTiles) return false;
  for (int c = 0; c < G; ++c)
    if (__builtin_popcountll(kb_mask_of(n_out, K, ks, c, G)) > kRegionSlots) return false;
  return true;
}

size_t action_block_ws_floats(int max_units) { return 2 * (size_t)max_units * BN * BM; }
size_t action_block_attn_ws_floats(int B, int H, int splits) { return (size_t)B * H * splits * kAttnPart; }
int action_block_cnt_ints() { return kCntInts; }

void action_block_attn_plan(int Lk, int bh, int nsm, int* splits, int* keys) {
  const int kb = (Lk + 63) / 64;  // 64-key blocks
  const int min_splits = (Lk + kActionBlockMaxKeys - 1) / kActionBlockMaxKeys;
  int s = bh > 0 ? nsm / bh : 1;  // one unit per SM where the heads allow it
  if (s > kb) s = kb;
  if (s < min_splits) s = min_splits;
  if (s > kMaxSplits) s = kMaxSplits;
  if (s < 1) s = 1;
  const int kps = ((kb + s - 1) / s) * 64;
  *keys = kps;
  *splits = (Lk + kps - 1) / kps;
}

cudaError_t prepare_action_block() {
  return cudaFuncSetAttribute(action_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
}

#ifdef WAM_AB_PHASES
extern "C" int wam_debug_ab_phases(unsigned long long* host) {
  return cudaMemcpyFromSymbol(host, g_ab_phase, sizeof g_ab_phase) == cudaSuccess ? 0 : 1;
}
#endif

cudaError_t launch_action_block(const ActionBlockMaps& m, const ActionBlockArgs& a, int ctas, cudaStream_t s) {
  if (ctas < 1 || a.n_gemm < 1 || a.n_gemm > kPh || a.Ma > BN || a.da % BM || a.da / BM > kMaxTiles ||
      (a.has_attn && (a.at.keys < 64 || a.at.keys > kActionBlockMaxKeys || a.at.keys % 64 ||
                      a.at.splits > kMaxSplits || a.La > BN)))
    return cudaErrorInvalidValue;
  return launch_k(action_block_kernel, dim3(ctas), dim3(kThr), kSmem, s, m, a);
}

}  // namespace wam
