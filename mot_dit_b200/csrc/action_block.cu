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
// Inside a launch the phases are separated by a grid-wide barrier (at most one
// CTA per SM and never more CTAs than SMs, so the whole grid is resident).
// Each GEMM phase is a fixed set of work units -- 128 weight rows x a fixed
// k-range -- chosen from the shapes and the SM count, never from the grid
// size; CTA c takes units c, c + G, ...  The MMA is tcgen05.mma with the
// weight rows on the 128 TMEM lanes and the tokens as the N = 32 operand, fp32
// accumulation in TMEM.  When a tile's k-range is split, every unit publishes
// its fp32 partial, and once all have, unit s sums token slice s of the tile
// over the splits in split order and applies the epilogue: the result depends
// neither on the grid size nor on timing, so every schedule is bitwise equal.
//
// Warp roles (192 threads):
//   warp 0     weight producer: one thread streams every weight k-block of the
//              launch (all phases, in order) through a TMA ring.  Weights do
//              not depend on the barriers, so the next phase's tiles are in
//              flight while the grid waits.
//   warp 1     TMEM owner and MMA issuer (one thread).
//   warps 2-5  compute: grid barriers, the B operand of each phase (TMA loads
//              of the activations, or the RMSNorm / AdaLN modulation of x_a
//              written straight into the swizzled operand layout), the
//              attention softmax and combine, the split reductions, epilogues.
//
// Attention of action block i over the joint keys [K^v_i; K^a_i] (rows
// [0, L_v + L_a) of the block's cache; summary page, 前置知识
// "Mixture-of-Transformers"): units are (sample, head, 128-key split).  S =
// Q K^T is one M = 128 MMA (the <= 32 queries padded with zero rows by the
// TMA fill), the thread of query q reads its 128 scores from TMEM and writes P
// (bf16) into the K-major operand tile over Q and K, and O = P V accumulates
// in TMEM with V as the MN-major operand.  Each unit publishes (row maximum,
// row sum, O); once all splits of a (sample, head) are in, split s combines
// query rows [q_s, q_s + ceil(L_a / splits)) in split order.
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
constexpr int kRegionSlots = 12;                // B k-blocks held at once
constexpr int kRegion = kRegionSlots * kBBlk;   // 48 KB (also Q | K | V of one attention unit)
constexpr int kStgLd = BM + 1;
constexpr int kStg = BN * kStgLd * 4;           // [32 tokens][129] fp32 staging
constexpr int kBarBytes = 256;
constexpr int kSmem = kStages * kTileA + kRegion + kStg + kBarBytes;
constexpr int kTmemCols = 256;                  // acc[2] at 0 / 32, S at 64..191, O at 192..255
constexpr int kKeys = 128;                      // keys per attention unit
constexpr int kMaxTiles = 64;                   // weight tiles of one phase (n_out <= 8192)
constexpr int kAttnPart = BN * 64 + 2 * BN;     // one attention partial: O [32][64], m [32], l [32]
constexpr int kMaps = kActionBlockMaps;


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

// 32 lanes x 64 consecutive 32-bit TMEM columns, one wait.
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
    __nanosleep(64);
  }
  return true;
}

// Grid-wide barrier of the compute warps (the producer and MMA threads touch
// no data that crosses CTAs).  Generation-based: the last arrival resets the
// count and bumps the generation, so the state is clean for the next barrier
// and the next launch.  Returns false when this CTA is winding down.
__device__ __forceinline__ bool grid_barrier(int* count, int* gen, int G, unsigned* status, volatile int* abort_flag) {
  bar_compute();
  if (threadIdx.x == 64 && !*abort_flag) {
    const volatile int* vg = gen;
    __threadfence();
    const int g0 = *vg;
    const int arrived = atomicAdd(count, 1);
    if (arrived == G - 1) {
      atomicExch(count, 0);
      __threadfence();
      atomicAdd(gen, 1);
    } else {
      const unsigned long long t0 = globaltimer();
      while (*vg == g0) {
        if (globaltimer() - t0 > kWaitLimitNs) {
          atomicOr(status, kStatusTimeoutPeer);
          *abort_flag = 1;
          break;
        }
        __nanosleep(32);
      }
    }
    __threadfence();
  }
  bar_compute();
  return !*abort_flag;
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
using APh = ActionAttnPhase;
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

// Epilogue of a slice of one tile, run by all 128 compute threads: the thread
// owns feature n = tile * 128 + f and v[j] = sum (bias not added) for token
// m0 + j, j < nm.  QKV items (64 features of one token per head) go through
// the staging buffer; every thread reaches its named barriers.
__device__ __forceinline__ void epilogue(const ActArgs& a, const GPh& p, int tile, int f, int m0, int nm,
                                         const float (&v)[32], float* stg) {
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
  if (!n_ok) return;
  switch (p.epi) {
    case kEpiGateRes: {
      const float g = __ldg(p.gate + n);
      float xo[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) xo[j] = j < nm ? __ldcg(p.out_f32 + (size_t)(m0 + j) * p.ld_out + n) : 0.f;
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j < nm) p.out_f32[(size_t)(m0 + j) * p.ld_out + n] = xo[j] + g * (v[j] + b);
      break;
    }
    case kEpiGelu:
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (j >= nm) break;
        p.out_act[(size_t)(m0 + j) * p.ld_out + n] = __float2bfloat16_rn(gelu_tanh(v[j] + b));
      }
      break;
    case kEpiStoreF32:
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (j >= nm) break;
        p.out_f32[(size_t)(m0 + j) * p.ld_out + n] = v[j] + b;
      }
      break;
    case kEpiEuler: {
      const float dt = a.aio->sched[p.step] - a.aio->sched[p.step + 1];
      float ao[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) ao[j] = j < nm ? __ldcg(p.out_f32 + (size_t)(m0 + j) * p.ld_out + n) : 0.f;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (j >= nm) break;
        const float an = ao[j] - dt * (v[j] + b);
        p.out_f32[(size_t)(m0 + j) * p.ld_out + n] = an;
        if (p.a_next) p.a_next[(size_t)(m0 + j) * p.a_next_ld + n] = __float2bfloat16_rn(an);
      }
      break;
    }
    default:
      break;
  }
}

__global__ void __launch_bounds__(kThr, 1)
    action_block_kernel(const __grid_constant__ ActMaps maps, const __grid_constant__ ActArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023) {
    if (threadIdx.x == 0) atomicOr(a.status, kStatusTimeoutDrain);
    return;
  }
  uint8_t* ring = smem_raw;                   // [kStages][16 KB] weight k-blocks
  uint8_t* region = ring + kStages * kTileA;  // 48 KB: B k-blocks, or Q | K | V (P over Q | K)
  float* stg = reinterpret_cast<float*>(region + kRegion);
  uint64_t* bars = reinterpret_cast<uint64_t*>(region + kRegion + kStg);
  uint64_t* full = bars;             // [kStages] weight k-block landed
  uint64_t* empty = full + kStages;  // [kStages] weight k-block read by the MMAs
  uint64_t* accf = empty + kStages;  // [2] accumulator ready
  uint64_t* acce = accf + 2;         // [2] accumulator drained (one arrival per compute warp)
  uint64_t* bready = acce + 2;       // B operand of a GEMM phase in place
  uint64_t* kvfull = bready + 1;     // Q, K, V of an attention unit landed
  uint64_t* sfull = kvfull + 1;      // S computed
  uint64_t* pfull = sfull + 1;       // P written (32 softmax threads)
  uint64_t* ofull = pfull + 1;       // O computed (P and V read)
  uint64_t* mdone = ofull + 1;       // every MMA of this CTA complete (teardown)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mdone + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int n_attn_units = a.has_attn ? a.B * a.H * a.at.splits : 0;

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
      for (int u = cta; u < n_attn_units && ok; u += G, ++ua) {
        if (!mbar_wait(kvfull, ua & 1, a.status, kStatusTimeoutTmaFull, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t q0 = smem_u32(region), k0 = q0 + 16384, v0 = q0 + 32768;
        constexpr uint32_t idesc_s = idesc_bf16_f32(128, kKeys);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 64) | (1u << 16);  // B (V) MN-major
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc_mma_bf16(tmem + 64, smem_desc_k128(q0 + k * 32), smem_desc_k128(k0 + k * 32), idesc_s, k > 0 ? 1u : 0u);
        tc_commit(sfull);
        issued = true;
        if (!mbar_wait(pfull, ua & 1, a.status, kStatusTimeoutAccum, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // P: two 64-key K-major tiles [128 rows][128 B] at q0 and q0 + 16 KB
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk)
          tc_mma_bf16(tmem + 192, smem_desc_k128(q0 + (kk >> 2) * 16384 + (kk & 3) * 32),
                      desc_mn128(v0 + kk * 16 * 128), idesc_pv, kk > 0 ? 1u : 0u);
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
            const uint32_t b0 = smem_u32(region + slot_of(mask, kb) * kBBlk);
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

    // ---------------- attention of the block
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
            mbar_arrive_expect_tx(kvfull, 3 * 16384);
            tma_load_3d(region, &maps.m[9], kvfull, 0, 0, bh);
            tma_load_3d(region + 16384, &maps.m[10], kvfull, 0, sp * kKeys, a.at.zk0 + bh);
            tma_load_3d(region + 32768, &maps.m[10], kvfull, 0, sp * kKeys, a.at.zv0 + bh);
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
          const int nvalid = min(kKeys, a.Lk - sp * kKeys);
          const uint32_t t_s = tmem + 64, t_o = tmem + 192;
          bool got = mbar_wait(sfull, ua & 1, a.status, kStatusTimeoutAccum, abort_flag);
          got = __all_sync(0xffffffffu, got) != 0;
          float mref = -INFINITY, lsum = 0.f;
          if (got) {
            tc_fence_after();
            float v[64];
            float mx = -INFINITY;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              tmem_ld64(t_s + 64 * half, v);
#pragma unroll
              for (int i = 0; i < 64; ++i)
                if (64 * half + i < nvalid) mx = fmaxf(mx, v[i]);
            }
            mref = mx * sl2e;
            uint8_t* prow = region + lane * 128;
            const int swz = lane & 7;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              tmem_ld64(t_s + 64 * half, v);
#pragma unroll
              for (int i = 0; i < 64; ++i) {
                const float pv = (64 * half + i < nvalid) ? ex2f(fmaf(v[i], sl2e, -mref)) : 0.f;
                v[i] = pv;
                lsum += pv;
              }
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                uint4 w;
                w.x = pack_bf16(v[8 * q + 0], v[8 * q + 1]);
                w.y = pack_bf16(v[8 * q + 2], v[8 * q + 3]);
                w.z = pack_bf16(v[8 * q + 4], v[8 * q + 5]);
                w.w = pack_bf16(v[8 * q + 6], v[8 * q + 7]);
                *reinterpret_cast<uint4*>(prow + half * 16384 + ((q ^ swz) << 4)) = w;
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
            __threadfence();
            __syncwarp();
            if (lane == 0) atomicAdd(a.cnt_attn + bh, 1);
          } else {
            *abort_flag = 1;
          }
        }
        bar_compute();
        if (*abort_flag) {
          ok = false;
          break;
        }
      }
      AB_STAMP(2);
      // combine: split sp of (sample, head) bh writes query rows [sp*qper, +qper)
      const int qper = (a.La + a.at.splits - 1) / a.at.splits;
      for (int u = cta; u < n_attn_units && ok; u += G) {
        const int bh = u / a.at.splits, sp = u % a.at.splits;
        const int q0 = sp * qper, nq = max(0, min(qper, a.La - q0));
        if (te == 0) wait_geq(a.cnt_attn + bh, a.at.splits, a.status, abort_flag);
        bar_compute();
        if (*abort_flag) {
          ok = false;
          break;
        }
        __threadfence();
        const int S2 = a.at.splits;
        const float* base = a.ws_attn + (size_t)bh * S2 * kAttnPart;
        const int bidx = bh / a.H, h = bh % a.H;
        // O rows [S2][nq][64] into the region by cp.async, (m, l) [S2][nq]
        // into the staging by plain loads: one round trip for all of them
        float* so = reinterpret_cast<float*>(region);
        float* sml = stg;  // [S2 * nq] m, then [S2 * nq] l
        for (int i = te; i < S2 * nq * 16; i += 128) {
          const int s2 = i / (nq * 16), rem = i - s2 * (nq * 16);
          cp_async16(smem_u32(so + 4 * i), base + (size_t)s2 * kAttnPart + q0 * 64 + 4 * rem, true);
        }
        cp_async_commit();
        if (te < S2 * nq) {
          const int s2 = te / nq, q = te - s2 * nq;
          const float* ps = base + (size_t)s2 * kAttnPart + BN * 64;
          const float mv = __ldcg(ps + q0 + q), lv = __ldcg(ps + BN + q0 + q);
          sml[te] = mv;
          sml[S2 * nq + te] = lv;
        }
        cp_async_wait<0>();
        bar_compute();
        for (int it = te; it < nq * 64; it += 128) {
          const int q = it / 64, d = it % 64;
          float M = -INFINITY;
          for (int s2 = 0; s2 < S2; ++s2) M = fmaxf(M, sml[s2 * nq + q]);
          float den = 0.f, acc = 0.f;
          for (int s2 = 0; s2 < S2; ++s2) {
            const float f = ex2f(sml[s2 * nq + q] - M);
            den += f * sml[S2 * nq + s2 * nq + q];
            acc += f * so[(s2 * nq + q) * 64 + d];
          }
          a.at.out[(size_t)(bidx * a.La + q0 + q) * a.at.ld_out + h * 64 + d] = __float2bfloat16_rn(acc / den);
        }
        bar_compute();
        if (te == 0) {
          __threadfence();
          if (atomicAdd(a.cnt_attn + a.B * a.H + bh, 1) == a.at.splits - 1) {
            a.cnt_attn[bh] = 0;
            a.cnt_attn[a.B * a.H + bh] = 0;
          }
        }
      }
    }

    // ---------------- GEMM phases
    AB_STAMP(3);
    int lt = 0;
    for (int pi = 0; pi < a.n_gemm && ok; ++pi) {
      const GPh& p = a.g[pi];
      if ((pi > 0 || n_attn_units > 0) && !grid_barrier(a.bar, a.bar + 1, G, a.status, abort_flag)) {
        ok = false;
        break;
      }
      AB_STAMP(4 + 4 * pi);
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
        // rms(x_a) (gain | 1 + scale) + shift, bf16, in the swizzled K-major layout
        const int r = te >> 2, part = te & 3;
        const bool valid = r < a.Ma;
        const float4* xr = reinterpret_cast<const float4*>(a.x_a + (size_t)(valid ? r : 0) * a.da);
        float ss = 0.f;
        const int n4 = a.da / 4;
        for (int i0 = part; i0 < n4; i0 += 4 * 12) {  // 12 loads in flight at a time
          float4 x4[12];
#pragma unroll
          for (int k = 0; k < 12; ++k) {
            const int i = i0 + 4 * k;
            x4[k] = i < n4 ? __ldcg(xr + i) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int k = 0; k < 12; ++k) ss += x4[k].x * x4[k].x + x4[k].y * x4[k].y + x4[k].z * x4[k].z + x4[k].w * x4[k].w;
        }
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        ss += __shfl_xor_sync(0xffffffffu, ss, 2);
        const float rr = 1.0f / sqrtf(ss / (float)a.da + 1e-6f);
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
        fence_async_smem();
        bar_compute();
        if (te == 0) {
          arrive(bready);
          bready_last = pi;
          bready_last_tma = false;
        }
      }
      AB_STAMP(5 + 4 * pi);
      // the units: accumulate, then finish (whole k-range) or publish (k-split)
      const int U = units_of(p);
      for (int u = cta; u < U; u += G, ++lt) {
        const int buf = lt & 1;
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
        const int t = u / p.ks;
        if (p.ks == 1) {
          epilogue(a, p, t, row, 0, a.Ma, v, stg);
        } else {
          float* part = a.ws + (size_t)u * (BN * BM);
#pragma unroll
          for (int j = 0; j < 32; ++j) __stcg(part + j * BM + row, v[j]);
          __threadfence();
          bar_compute();
          if (te == 0) atomicAdd(a.cnt + t, 1);
        }
      }
      AB_STAMP(6 + 4 * pi);
      if (!ok || p.ks == 1) continue;
      // split reduction: unit (t, s) sums token slice s of tile t over the splits, in order
      const int per = (a.Ma + p.ks - 1) / p.ks;
      for (int u = cta; u < U; u += G) {
        const int t = u / p.ks, s = u % p.ks;
        const int m0 = s * per, nm = max(0, min(per, a.Ma - m0));
        if (te == 0) wait_geq(a.cnt + t, p.ks, a.status, abort_flag);
        bar_compute();
        if (*abort_flag) {
          ok = false;
          break;
        }
        __threadfence();
        // every split's slice [nm tokens][128 features] into the region (free:
        // this CTA's MMAs of the phase are complete), all copies in flight at
        // once, then the sums in split order from shared memory
        float* red = reinterpret_cast<float*>(region);  // [ks][nm][128]
        const int n16 = p.ks * nm * (BM / 4);
        for (int i = te; i < n16; i += 128) {
          const int s2 = i / (nm * (BM / 4)), rem = i - s2 * (nm * (BM / 4));
          cp_async16(smem_u32(red + 4 * i), a.ws + ((size_t)(t * p.ks + s2) * BN + m0) * BM + 4 * rem, true);
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
        epilogue(a, p, t, te, m0, nm, v, stg);
        bar_compute();
        if (te == 0) {
          __threadfence();
          if (atomicAdd(a.cnt + kMaxTiles + t, 1) == p.ks - 1) {
            a.cnt[t] = 0;
            a.cnt[kMaxTiles + t] = 0;
          }
        }
      }
      AB_STAMP(7 + 4 * pi);
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
  if (K % BK || K / BK > 64) return false;
  for (int c = 0; c < G; ++c)
    if (__builtin_popcountll(kb_mask_of(n_out, K, ks, c, G)) > kRegionSlots) return false;
  return true;
}

size_t action_block_ws_floats(int max_units) { return (size_t)max_units * BN * BM; }
size_t action_block_attn_ws_floats(int B, int H, int splits) { return (size_t)B * H * splits * kAttnPart; }
int action_block_attn_splits(int Lk) { return (Lk + kKeys - 1) / kKeys; }

cudaError_t prepare_action_block() {
  return cudaFuncSetAttribute(action_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
}

#ifdef WAM_AB_PHASES
extern "C" int wam_debug_ab_phases(unsigned long long* host) {
  return cudaMemcpyFromSymbol(host, g_ab_phase, sizeof g_ab_phase) == cudaSuccess ? 0 : 1;
}
#endif

cudaError_t launch_action_block(const ActionBlockMaps& m, const ActionBlockArgs& a, int ctas, cudaStream_t s) {
  if (ctas < 1 || a.n_gemm < 1 || a.n_gemm > 5 || a.Ma > BN || a.da % BK) return cudaErrorInvalidValue;
  return launch_k(action_block_kernel, dim3(ctas), dim3(kThr), kSmem, s, m, a);
}

}  // namespace wam
