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
// Persistent: each CTA walks a static, strided list of work units (tile x
// split), so the schedule -- and every reduction order -- is a function of the
// launch configuration only.  The accumulator is double-buffered in TMEM
// (2 x BN columns): the MMA warp fills buffer b of unit j+1 while the epilogue
// warps drain buffer b^1 of unit j.
//
// Orientation.  Normal: A = X (128 tokens on TMEM lanes), B = W (BN features).
// Swapped (few tokens, e.g. the action expert's 32): A = W (128 features on
// TMEM lanes), B = X (BN tokens) -- the weight stream fills the 128-row MMA
// operand instead of padding the token dimension.
//
// Split-K (swapped only): each unit reduces a K range into TMEM and writes an
// fp32 partial tile; the last unit of a tile (integer ticket) sums the
// partials in split order 0..S-1 -- a fixed order, so the result does not
// depend on which CTA finishes last.
//
// Epilogue stores are coalesced: a 32 x 32 sub-tile held one-row-per-thread
// after tcgen05.ld goes through padded shared memory and is written one row
// per warp instruction (32 consecutive columns), except the QK-norm + RoPE
// epilogue, which keeps a head's 64 channels in one thread.
//
// Warp roles (192 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA
// issuer, warps 2..5 epilogue (warp w reads TMEM lanes 32*(w%4) .. +31).
#include <cstdio>

#include "common.cuh"
#include "kernels.h"

namespace wam {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kThreads = 192;

template <int BN, bool SWAP>
struct TileCfg {
  static constexpr int kABytes = BM * BK * 2;
  static constexpr int kBBytes = BN * BK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = 2 * BN <= 32 ? 32 : (2 * BN <= 64 ? 64 : (2 * BN <= 128 ? 128 : (2 * BN <= 256 ? 256 : 512)));
  // Normal orientation, BN <= 128: each epilogue warp prefetches its 32 x BN
  // residual rows (gate-residual) or 32 RoPE rows (QKV) while the MMA runs.
  static constexpr bool kPrefetch = !SWAP && BN <= 128;
  static constexpr int kResBytes = kPrefetch ? 4 * 32 * BN * 4 : 0;
  // Swapped orientation: [32 tokens][128 features + 1] fp32 staging of the QKV epilogue.
  static constexpr int kEpiBytes = SWAP ? 32 * (BM + 1) * 4 : 0;
  static constexpr int kBarBytes = 256;
  static constexpr int kSmemMax = 232448;  // 227 KB per CTA
  static constexpr int kFit = (kSmemMax - 1024 - kBarBytes - kResBytes - kEpiBytes) / kStageBytes;
  static constexpr int kStages = kFit > 8 ? 8 : kFit;  // deep ring: TMA latency > a few MMA k-blocks
  static constexpr int kSmem = kStages * kStageBytes + kEpiBytes + kResBytes + kBarBytes + 1024;
  static_assert(kStages >= 3, "shared memory ring too shallow");
};

struct GemmK {
  int rows_a, rows_b, K;
  int z_a, z_b;
  int tiles_a, tiles_b;
  int kb_per_split, splits;
  int units;
  float* ws;
  int* tickets;
  unsigned* status;
};

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ void store_act(void* base, size_t idx, float v) {
  reinterpret_cast<__nv_bfloat16*>(base)[idx] = __float2bfloat16_rn(v);
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
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
  return r;
}

// Per-head QK-RMSNorm (gain), RoPE, and scatter of one 64-channel head vector
// of token m.  section: 0 = q, 1 = k, 2 = v.  cs_row / sn_row: the token's
// cos / sin row, prefetched in shared memory with its 16-byte chunks permuted
// by XOR with swz (or null to read the table).
__device__ __forceinline__ void qkv_emit(const EpiRegs& R, int section, int head, int m, float (&x)[64],
                                         const float* cs_row = nullptr, const float* sn_row = nullptr,
                                         int swz = 0) {
  const int b = m / R.seq_len, l = m - b * R.seq_len;
  if (section < 2) {
    const float4* g4 = reinterpret_cast<const float4*>((section == 0 ? R.gq : R.gk) + head * 64);
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < 64; ++j) ss += x[j] * x[j];
    const float r = rsqrtf(ss * (1.0f / 64.0f) + 1e-6f);
#pragma unroll
    for (int j4 = 0; j4 < 16; ++j4) {
      const float4 gg = __ldg(g4 + j4);
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
  __nv_bfloat16* dst;
  if (section == 0)
    dst = R.q_out + ((size_t)(b * R.n_heads + head) * R.seq_len + l) * 64;
  else
    dst = (section == 1 ? R.k_cache : R.v_cache) + ((size_t)(b * R.n_heads + head) * R.cache_len + R.cache_off + l) * 64;
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
      store_act(e.out_act, idx, gelu_tanh(y));
      break;
    case kEpiEuler: {
      const float dt = e.aio->sched[e.step] - e.aio->sched[e.step + 1];
      const float a = e.out_f32[idx] - dt * y;
      e.out_f32[idx] = a;
      if (e.a_next) store_act(e.a_next, (size_t)m * e.a_next_ld + n, a);
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
    default:
      break;
  }
}

template <int BN, bool SWAP>
__global__ void __launch_bounds__(kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                   const GemmK g, const EpiArgs e) {
  using C = TileCfg<BN, SWAP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::kStages * C::kABytes;
  float* sEpi = reinterpret_cast<float*>(smem + C::kStages * C::kStageBytes);  // swapped QKV staging
  float* sRes = reinterpret_cast<float*>(smem + C::kStages * C::kStageBytes + C::kEpiBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes + C::kEpiBytes + C::kResBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* accf = empty + C::kStages;  // [2] accumulator ready (MMA -> epilogue)
  uint64_t* acce = accf + 2;            // [2] accumulator drained (epilogue -> MMA)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kb_total = (g.K + BK - 1) / BK;
  const int per_tile_units = g.splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], 4);
    }
    *abort_flag = 0;
    *last_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&map_a);
    prefetch_tensormap(&map_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();  // the next kernel may start its own set-up now

  // unit u -> (tile_a, tile_b, split); split fastest, then tile_a, then tile_b
  auto decode = [&](int u, int& ta, int& tb, int& sp) {
    sp = u % per_tile_units;
    const int t = u / per_tile_units;
    ta = t % g.tiles_a;
    tb = t / g.tiles_a;
  };

  if (warp == 0) {
    if (lane == 0) {
      int it = 0, issued = 0;
      bool ok = true;
      // The weights never change during a chunk: the first unit's weight tiles
      // are requested before waiting for the previous kernel (dependent launch).
      int pre = 0;
      if (blockIdx.x < g.units) {
        int ta, tb, sp;
        decode(blockIdx.x, ta, tb, sp);
        const int kb0 = sp * g.kb_per_split, kb1 = min(kb_total, kb0 + g.kb_per_split);
        pre = min(C::kStages, kb1 - kb0);
        for (int i = 0; i < pre; ++i) {
          mbar_arrive_expect_tx(&full[i], C::kStageBytes);
          if (SWAP)
            tma_load_3d(sA + i * C::kABytes, &map_a, &full[i], (kb0 + i) * BK, ta * BM, g.z_a);
          else
            tma_load_3d(sB + i * C::kBBytes, &map_b, &full[i], (kb0 + i) * BK, tb * BN, g.z_b);
        }
        pdl_wait();
        for (int i = 0; i < pre; ++i) {
          if (SWAP)
            tma_load_3d(sB + i * C::kBBytes, &map_b, &full[i], (kb0 + i) * BK, tb * BN, g.z_b);
          else
            tma_load_3d(sA + i * C::kABytes, &map_a, &full[i], (kb0 + i) * BK, ta * BM, g.z_a);
        }
        issued = pre;
      } else {
        pdl_wait();
      }
      for (int u = blockIdx.x; u < g.units && ok; u += gridDim.x) {
        int ta, tb, sp;
        decode(u, ta, tb, sp);
        const int kb0 = sp * g.kb_per_split, kb1 = min(kb_total, kb0 + g.kb_per_split);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          if (it < pre) continue;  // issued above
          const int s = it % C::kStages;
          if (it >= C::kStages &&
              !mbar_wait(&empty[s], ((it / C::kStages) - 1) & 1, g.status, kStatusTimeoutTmaEmpty, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], C::kStageBytes);
          tma_load_3d(sA + s * C::kABytes, &map_a, &full[s], kb * BK, ta * BM, g.z_a);
          tma_load_3d(sB + s * C::kBBytes, &map_b, &full[s], kb * BK, tb * BN, g.z_b);
          issued = it + 1;
        }
      }
      // Drain: never leave the CTA with copies into its shared memory in flight.
      for (int i = max(0, issued - C::kStages); i < issued; ++i)
        mbar_wait(&full[i % C::kStages], (i / C::kStages) & 1, g.status, kStatusTimeoutDrain, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN);
      int it = 0, lt = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < g.units && ok; u += gridDim.x, ++lt) {
        int ta, tb, sp;
        decode(u, ta, tb, sp);
        const int kb0 = sp * g.kb_per_split, kb1 = min(kb_total, kb0 + g.kb_per_split);
        const int buf = lt & 1;
        if (lt >= 2 && !mbar_wait(&acce[buf], ((lt >> 1) - 1) & 1, g.status, kStatusTimeoutAccum, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + buf * BN;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % C::kStages;
          if (!mbar_wait(&full[s], (it / C::kStages) & 1, g.status, kStatusTimeoutTmaFull, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * C::kABytes);
          const uint32_t b0 = smem_u32(sB + s * C::kBBytes);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            tc_mma_bf16(d_tmem, smem_desc_k128(a0 + k * 32), smem_desc_k128(b0 + k * 32), idesc,
                        (kb > kb0 || k > 0) ? 1u : 0u);
          tc_commit(&empty[s]);
        }
        tc_commit(&accf[buf]);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    pdl_wait();  // outputs / residual rows belong to the previous kernel until it is done
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const EpiRegs R = hoist(e);
    float* res = sRes + quad * (32 * BN);  // this warp's prefetched residual rows / RoPE rows
    constexpr bool kRopeFits = C::kPrefetch && BN >= 64;  // 32 cos + 32 sin rows of 32 floats
    int lt = 0;
    for (int u = blockIdx.x; u < g.units; u += gridDim.x, ++lt) {
      int ta, tb, sp;
      decode(u, ta, tb, sp);
      const int buf = lt & 1;
      bool prefetched = false;
      if constexpr (C::kPrefetch) {
        // While the MMA of this unit runs: bring this warp's residual rows
        // (16-byte chunk q of row r at chunk q ^ (r & 7): thread-per-row
        // reads are then conflict-free) or its tokens' RoPE rows into smem.
        const int m0 = ta * BM + quad * 32, nb = tb * BN;
        if (R.kind == kEpiGateRes) {
          for (int k = lane; k < 32 * (BN / 4); k += 32) {
            const int r = k / (BN / 4), q = k % (BN / 4);
            const int m = m0 + r, n = nb + 4 * q;
            const bool v = m < g.rows_a && n < g.rows_b;
            cp_async16(smem_u32(res + r * BN + 4 * (q ^ (r & 7))),
                       v ? (const void*)(R.out_f32 + (size_t)m * R.ld + n) : (const void*)R.out_f32, v);
          }
          cp_async_commit();
          prefetched = true;
        } else if (kRopeFits && R.kind == kEpiQkv) {
          for (int k = lane; k < 32 * 16; k += 32) {
            const int r = k >> 4, which = (k >> 3) & 1, c4 = k & 7;
            const int m = min(m0 + r, g.rows_a - 1);
            const int pos = R.cache_off + (m % R.seq_len);
            const float* src = (which ? R.rope_sin : R.rope_cos) + pos * 32 + 4 * c4;
            cp_async16(smem_u32(res + which * (32 * 32) + r * 32 + 4 * (c4 ^ (r & 7))), src, true);
          }
          cp_async_commit();
          prefetched = true;
        }
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
        if (lane == 0) mbar_arrive(&acce[buf]);
      };

      if (!SWAP) {
        // thread = output row m, 32 consecutive features per TMEM load
        const int m = ta * BM + quad * 32 + lane;
        const int nb = tb * BN;
        const bool m_ok = m < g.rows_a;
        if (R.kind == kEpiQkv) {
          for (int c = 0; c < BN; c += 64) {
            float x[64];
            float (&lo)[32] = *reinterpret_cast<float(*)[32]>(&x[0]);
            float (&hi)[32] = *reinterpret_cast<float(*)[32]>(&x[32]);
            tmem_ld32(t_row + c, lo);
            tmem_ld32(t_row + c + 32, hi);
            if (c + 64 >= BN) release();
            const int n = nb + c;
            if (m_ok && n < g.rows_b) {
              const float4* b4 = reinterpret_cast<const float4*>(R.bias + n);
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const float4 bb = __ldg(b4 + j);
                x[4 * j] += bb.x;
                x[4 * j + 1] += bb.y;
                x[4 * j + 2] += bb.z;
                x[4 * j + 3] += bb.w;
              }
              if constexpr (kRopeFits)
                qkv_emit(R, n / R.attn_dim, (n % R.attn_dim) / 64, m, x, res + lane * 32, res + 32 * 32 + lane * 32,
                         lane & 7);
              else
                qkv_emit(R, n / R.attn_dim, (n % R.attn_dim) / 64, m, x);
            }
          }
        } else {
          for (int c = 0; c < BN; c += 32) {
            float v[32];
            tmem_ld32(t_row + c, v);
            if (c + 32 >= BN) release();
            const int n0 = nb + c;
            if (!m_ok || n0 >= g.rows_b) continue;
            const float4* b4 = reinterpret_cast<const float4*>(R.bias + n0);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float4 bb = __ldg(b4 + j);
              v[4 * j] += bb.x;
              v[4 * j + 1] += bb.y;
              v[4 * j + 2] += bb.z;
              v[4 * j + 3] += bb.w;
            }
            if (R.kind == kEpiStoreF32) {
              float4* o = reinterpret_cast<float4*>(R.out_f32 + (size_t)m * R.ld + n0);
#pragma unroll
              for (int j = 0; j < 8; ++j) o[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            } else if (R.kind == kEpiGelu) {
              uint4* o = reinterpret_cast<uint4*>(R.out_act + (size_t)m * R.ld + n0);
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                uint4 w;
                w.x = pack_bf16(gelu_tanh(v[8 * j + 0]), gelu_tanh(v[8 * j + 1]));
                w.y = pack_bf16(gelu_tanh(v[8 * j + 2]), gelu_tanh(v[8 * j + 3]));
                w.z = pack_bf16(gelu_tanh(v[8 * j + 4]), gelu_tanh(v[8 * j + 5]));
                w.w = pack_bf16(gelu_tanh(v[8 * j + 6]), gelu_tanh(v[8 * j + 7]));
                o[j] = w;
              }
            } else if (R.kind == kEpiGateRes) {
              float4 xo[8];
              float4* o = reinterpret_cast<float4*>(R.out_f32 + (size_t)m * R.ld + n0);
              if (C::kPrefetch) {
#pragma unroll
                for (int j = 0; j < 8; ++j)
                  xo[j] = *reinterpret_cast<const float4*>(res + lane * BN + 4 * (((c >> 2) + j) ^ (lane & 7)));
              } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) xo[j] = o[j];
              }
              const float4* g4 = reinterpret_cast<const float4*>(R.gate + n0);
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const float4 gg = __ldg(g4 + j);
                o[j] = make_float4(xo[j].x + gg.x * v[4 * j], xo[j].y + gg.y * v[4 * j + 1],
                                   xo[j].z + gg.z * v[4 * j + 2], xo[j].w + gg.w * v[4 * j + 3]);
              }
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) epi_elem(e, m, n0 + j, v[j], 0.f);
            }
          }
        }
      } else {
        // swapped: TMEM lane = feature n, column = token
        const int n = ta * BM + row;
        const int mb = tb * BN;
        const int tile_lin = ta + g.tiles_a * tb;
        const bool n_ok = n < g.rows_a;
        const float bias = n_ok ? __ldg(R.bias + n) : 0.f;
        const float gate = (n_ok && R.gate) ? __ldg(R.gate + n) : 0.f;
        bool last = true;
        if (g.splits > 1) {
          float* my = g.ws + ((size_t)(tile_lin * g.splits + sp) * BM + row) * BN;
          for (int c = 0; c < BN; c += 32) {
            float v[32];
            tmem_ld32(t_row + c, v);
            if (c + 32 >= BN) release();
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              __stcg(reinterpret_cast<float4*>(my + c + j), make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]));
          }
          __threadfence();
          epi_bar();
          if (threadIdx.x == 64) {
            const int prev = atomicAdd(g.tickets + tile_lin, 1);
            *last_flag = (prev == g.splits - 1) ? 1 : 0;
          }
          epi_bar();
          last = *last_flag != 0;
          __threadfence();
        }
        if (last) {
          for (int c = 0; c < BN; c += 32) {
            float v[32];
            if (g.splits > 1) {
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = 0.f;
              const float* p = g.ws + ((size_t)(tile_lin * g.splits) * BM + row) * BN + c;
              const size_t sstride = (size_t)BM * BN;
              int s = 0;
              for (; s + 2 <= g.splits; s += 2) {  // two splits in flight, summed in split order
                float4 t0[8], t1[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                  t0[j] = __ldcg(reinterpret_cast<const float4*>(p + s * sstride) + j);
                  t1[j] = __ldcg(reinterpret_cast<const float4*>(p + (s + 1) * sstride) + j);
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                  v[4 * j] += t0[j].x;
                  v[4 * j + 1] += t0[j].y;
                  v[4 * j + 2] += t0[j].z;
                  v[4 * j + 3] += t0[j].w;
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                  v[4 * j] += t1[j].x;
                  v[4 * j + 1] += t1[j].y;
                  v[4 * j + 2] += t1[j].z;
                  v[4 * j + 3] += t1[j].w;
                }
              }
              for (; s < g.splits; ++s) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                  const float4 t4 = __ldcg(reinterpret_cast<const float4*>(p + s * sstride) + j);
                  v[4 * j] += t4.x;
                  v[4 * j + 1] += t4.y;
                  v[4 * j + 2] += t4.z;
                  v[4 * j + 3] += t4.w;
                }
              }
            } else {
              tmem_ld32(t_row + c, v);
              if (c + 32 >= BN) release();
            }
            if (R.kind == kEpiQkv) {
              // stage [32 tokens][128 features + 1] and emit (token, head) items
              float* stage = sEpi;
              epi_bar();  // previous chunk's readers are done with the stage
#pragma unroll
              for (int j = 0; j < 32; ++j) stage[j * (BM + 1) + row] = v[j] + bias;
              epi_bar();
              const int t = threadIdx.x - 64;
              if (t < 64) {
                const int j = t & 31, hh = t >> 5;
                const int m = mb + c + j;
                const int n0 = ta * BM + hh * 64;
                if (m < g.rows_b && n0 < g.rows_a) {
                  float x[64];
#pragma unroll
                  for (int k = 0; k < 64; ++k) x[k] = stage[j * (BM + 1) + hh * 64 + k];
                  qkv_emit(R, n0 / R.attn_dim, (n0 % R.attn_dim) / 64, m, x);
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
            } else if (n_ok) {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const int m = mb + c + j;
                if (m < g.rows_b) epi_elem(e, m, n, v[j] + bias, gate);
              }
            }
          }
          if (g.splits > 1 && threadIdx.x == 64) g.tickets[tile_lin] = 0;
        }
      }
    }
  }

  // ------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // wait for the last commits of this CTA's MMAs before freeing TMEM
    if (lane == 0) {
      int nloc = 0;
      for (int u = blockIdx.x; u < g.units; u += gridDim.x) ++nloc;
      for (int l = max(0, nloc - 2); l < nloc; ++l)
        mbar_wait(&accf[l & 1], (l >> 1) & 1, g.status, kStatusTimeoutDrain, nullptr);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int BN, bool SWAP>
cudaError_t prepare_bn() {
  return cudaFuncSetAttribute(tc_gemm_kernel<BN, SWAP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              TileCfg<BN, SWAP>::kSmem);
}

int g_num_sms = 0;

template <int BN, bool SWAP>
cudaError_t launch_bn(const TcGemm& t, const EpiArgs& e, cudaStream_t s) {
  using C = TileCfg<BN, SWAP>;
  GemmK g;
  g.rows_a = t.rows_a;
  g.rows_b = t.rows_b;
  g.K = t.K;
  g.z_a = t.z_a;
  g.z_b = t.z_b;
  const int kb_total = (t.K + BK - 1) / BK;
  int splits = t.swap ? (t.splits < 1 ? 1 : t.splits) : 1;
  if (splits > kb_total) splits = kb_total;
  g.kb_per_split = (kb_total + splits - 1) / splits;
  splits = (kb_total + g.kb_per_split - 1) / g.kb_per_split;  // no empty split
  g.splits = splits;
  g.tiles_a = (t.rows_a + BM - 1) / BM;
  g.tiles_b = (t.rows_b + BN - 1) / BN;
  g.units = g.tiles_a * g.tiles_b * splits;
  g.ws = t.ws;
  g.tickets = t.tickets;
  g.status = t.status;
  int ctas = t.max_ctas > 0 ? t.max_ctas : g_num_sms;
  if (ctas > g.units) ctas = g.units;
  if (ctas < 1) ctas = 1;
  return launch_k(tc_gemm_kernel<BN, SWAP>, dim3(ctas), dim3(kThreads), C::kSmem, s, *t.map_a, *t.map_b, g, e);
}

}  // namespace

cudaError_t prepare_tc_gemm() {
  cudaError_t e;
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = prepare_bn<32, true>()) != cudaSuccess) return e;
  if ((e = prepare_bn<64, true>()) != cudaSuccess) return e;
  if ((e = prepare_bn<128, true>()) != cudaSuccess) return e;
  if ((e = prepare_bn<256, true>()) != cudaSuccess) return e;
  if ((e = prepare_bn<64, false>()) != cudaSuccess) return e;
  if ((e = prepare_bn<96, false>()) != cudaSuccess) return e;
  if ((e = prepare_bn<128, false>()) != cudaSuccess) return e;
  return prepare_bn<256, false>();
}

cudaError_t launch_tc_gemm(const TcGemm& t, const EpiArgs& e, cudaStream_t s) {
  if (g_num_sms == 0) return cudaErrorNotReady;
  // the normal orientation's epilogue writes whole 32-feature groups
  if (!t.swap && t.rows_b % 32 != 0) return cudaErrorInvalidValue;
  if (t.swap) {
    switch (t.bn) {
      case 32: return launch_bn<32, true>(t, e, s);
      case 64: return launch_bn<64, true>(t, e, s);
      case 128: return launch_bn<128, true>(t, e, s);
      case 256: return launch_bn<256, true>(t, e, s);
    }
  } else {
    switch (t.bn) {
      case 64: return launch_bn<64, false>(t, e, s);
      case 96: return launch_bn<96, false>(t, e, s);
      case 128: return launch_bn<128, false>(t, e, s);
      case 256: return launch_bn<256, false>(t, e, s);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace wam
