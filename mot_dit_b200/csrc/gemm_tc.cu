// tcgen05 GEMM for sm_100a with the MoT block epilogues fused in.
//
// C[m, n] = sum_k X[m, k] W[n, k]: X = activations (tokens x K), W = a weight
// stored [out, in] (K contiguous).  Both operands are K-major bf16 tiles moved
// by TMA (128-byte swizzle) into a multi-stage shared-memory ring; one thread
// issues tcgen05.mma (M = 128, N = BN, K = 16) into an fp32 accumulator in
// tensor memory; four epilogue warps read it back with tcgen05.ld and apply
// the fused epilogue (bias, gate-residual, GELU, QK-norm + RoPE + K/V publish,
// Euler update).
//
// Orientation.  Normal: A = X (128 tokens on TMEM lanes), B = W (BN features).
// Swapped (few tokens, e.g. the action expert's 32): A = W (128 features on
// TMEM lanes), B = X (BN tokens) -- the weight stream fills the 128-row MMA
// operand instead of padding the token dimension.
//
// Split-K (swapped only): each CTA reduces a K range into TMEM, writes the
// fp32 partial tile, and the last CTA of a tile (integer ticket) sums the
// partials in split order 0..S-1 -- a fixed order, so the result does not
// depend on which CTA finishes last.
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

template <int BN>
struct TileCfg {
  static constexpr int kStages = BN >= 256 ? 4 : (BN >= 128 ? 5 : 4);
  static constexpr int kABytes = BM * BK * 2;
  static constexpr int kBBytes = BN * BK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = BN < 32 ? 32 : BN;
  static constexpr int kBarBytes = 256;
  static constexpr int kSmem = kStages * kStageBytes + kBarBytes + 1024;
};

struct GemmK {
  int rows_a, rows_b, K;
  int z_a, z_b;
  int kb_per_split, splits;
  float* ws;
  int* tickets;
  unsigned* status;
};

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ void store_act(void* base, size_t idx, float v) {
  reinterpret_cast<__nv_bfloat16*>(base)[idx] = __float2bfloat16_rn(v);
}

// Per-head QK-RMSNorm (gain), RoPE, and scatter of one 64-channel head vector
// of token m.  section: 0 = q, 1 = k, 2 = v.
__device__ __forceinline__ void qkv_emit(const EpiArgs& e, int section, int head, int m, float (&x)[64]) {
  const int b = m / e.seq_len, l = m - b * e.seq_len;
  if (section < 2) {
    const float* g = (section == 0 ? e.gq : e.gk) + head * 64;
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < 64; ++j) ss += x[j] * x[j];
    const float r = rsqrtf(ss * (1.0f / 64.0f) + 1e-6f);
#pragma unroll
    for (int j = 0; j < 64; ++j) x[j] *= r * __ldg(g + j);
    const int pos = e.cache_off + l;
    const float* cs = e.rope_cos + pos * 32;
    const float* sn = e.rope_sin + pos * 32;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float c = __ldg(cs + j), s = __ldg(sn + j);
      const float x1 = x[j], x2 = x[j + 32];
      x[j] = x1 * c - x2 * s;
      x[j + 32] = x1 * s + x2 * c;
    }
  }
  __nv_bfloat16* dst;
  if (section == 0) {
    dst = reinterpret_cast<__nv_bfloat16*>(e.q_out) + ((size_t)(b * e.n_heads + head) * e.seq_len + l) * 64;
  } else {
    __nv_bfloat16* c = reinterpret_cast<__nv_bfloat16*>(section == 1 ? e.k_cache : e.v_cache);
    dst = c + ((size_t)(b * e.n_heads + head) * e.cache_len + e.cache_off + l) * 64;
  }
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

// Elementwise epilogue of one value at (token m, feature n).
__device__ __forceinline__ void epi_elem(const EpiArgs& e, int m, int n, float acc) {
  const float y = acc + __ldg(e.bias + n);
  const size_t idx = (size_t)m * e.ld_out + n;
  switch (e.kind) {
    case kEpiStoreF32:
      e.out_f32[idx] = y;
      break;
    case kEpiGateRes:
      e.out_f32[idx] += __ldg(e.gate + n) * y;
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
  using C = TileCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::kStages * C::kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* accb = empty + C::kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accb + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile_a = blockIdx.x, tile_b = blockIdx.y, split = blockIdx.z;
  const int kb_total = (g.K + BK - 1) / BK;
  const int kb0 = split * g.kb_per_split;
  const int kb1 = min(kb_total, kb0 + g.kb_per_split);
  const int nkb = kb1 - kb0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accb, 1);
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

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nkb; ++i) {
        const int s = i % C::kStages;
        if (i >= C::kStages &&
            !mbar_wait(&empty[s], ((i / C::kStages) - 1) & 1, g.status, kStatusTimeoutTmaEmpty, abort_flag))
          break;
        mbar_arrive_expect_tx(&full[s], C::kStageBytes);
        const int kx = (kb0 + i) * BK;
        tma_load_3d(sA + s * C::kABytes, &map_a, &full[s], kx, tile_a * BM, g.z_a);
        tma_load_3d(sB + s * C::kBBytes, &map_b, &full[s], kx, tile_b * BN, g.z_b);
        issued = i + 1;
      }
      // Drain: never leave the CTA with copies into its shared memory in flight.
      for (int i = max(0, issued - C::kStages); i < issued; ++i)
        mbar_wait(&full[i % C::kStages], (i / C::kStages) & 1, g.status, kStatusTimeoutDrain, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN);
      for (int i = 0; i < nkb; ++i) {
        const int s = i % C::kStages;
        if (!mbar_wait(&full[s], (i / C::kStages) & 1, g.status, kStatusTimeoutTmaFull, abort_flag)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + s * C::kABytes);
        const uint32_t b0 = smem_u32(sB + s * C::kBBytes);
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)
          tc_mma_bf16(tmem, smem_desc_k128(a0 + k * 32), smem_desc_k128(b0 + k * 32), idesc,
                      (i > 0 || k > 0) ? 1u : 0u);
        tc_commit(&empty[s]);
      }
      tc_commit(accb);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t t_row = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const bool ok = mbar_wait(accb, 0, g.status, kStatusTimeoutAccum, abort_flag);
    tc_fence_after();
    if (!ok) *abort_flag = 1;
    // One decision for all four epilogue warps: every later named barrier is
    // reached by all of them or by none.  The MMA warp has committed (or given
    // up) by now and the producer only drains, so the flag no longer changes.
    epi_bar();
    if (!*abort_flag) {
      if (!SWAP) {
        const int m = tile_a * BM + row;
        const int nb = tile_b * BN;
        if (e.kind == kEpiQkv) {
          for (int c = 0; c < BN; c += 64) {
            float x[64];
            float (&lo)[32] = *reinterpret_cast<float(*)[32]>(&x[0]);
            float (&hi)[32] = *reinterpret_cast<float(*)[32]>(&x[32]);
            tmem_ld32(t_row + c, lo);
            tmem_ld32(t_row + c + 32, hi);
            const int n = nb + c;
            if (m < g.rows_a && n < g.rows_b) {
#pragma unroll
              for (int j = 0; j < 64; ++j) x[j] += __ldg(e.bias + n + j);
              qkv_emit(e, n / e.attn_dim, (n % e.attn_dim) / 64, m, x);
            }
          }
        } else {
          for (int c = 0; c < BN; c += 32) {
            float v[32];
            tmem_ld32(t_row + c, v);
            if (m < g.rows_a) {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const int n = nb + c + j;
                if (n < g.rows_b) epi_elem(e, m, n, v[j]);
              }
            }
          }
        }
      } else {
        // swapped: TMEM lane = feature, column = token
        const int n = tile_a * BM + row;
        const int mb = tile_b * BN;
        const int tile_lin = tile_a + gridDim.x * tile_b;
        bool last = true;
        if (g.splits > 1) {
          float* my = g.ws + ((size_t)(tile_lin * g.splits + split) * BM + row) * BN;
          for (int c = 0; c < BN; c += 32) {
            float v[32];
            tmem_ld32(t_row + c, v);
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              *reinterpret_cast<float4*>(my + c + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
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
          float* stage = reinterpret_cast<float*>(smem);  // [BN][BM + 1] (pipeline ring is idle now)
          for (int c = 0; c < BN; c += 32) {
            float v[32];
            if (g.splits > 1) {
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = 0.f;
              for (int s = 0; s < g.splits; ++s) {
                const float* p = g.ws + ((size_t)(tile_lin * g.splits + s) * BM + row) * BN + c;
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                  const float4 t4 = __ldcg(reinterpret_cast<const float4*>(p + j));
                  v[j] += t4.x;
                  v[j + 1] += t4.y;
                  v[j + 2] += t4.z;
                  v[j + 3] += t4.w;
                }
              }
            } else {
              tmem_ld32(t_row + c, v);
            }
            if (e.kind == kEpiQkv) {
              const float bn_ = (n < g.rows_a) ? __ldg(e.bias + n) : 0.f;
#pragma unroll
              for (int j = 0; j < 32; ++j) stage[(c + j) * (BM + 1) + row] = v[j] + bn_;
            } else if (n < g.rows_a) {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const int m = mb + c + j;
                if (m < g.rows_b) epi_elem(e, m, n, v[j]);
              }
            }
          }
          if (e.kind == kEpiQkv) {
            epi_bar();
            // items: (token j, head hh) for the two heads of this 128-feature tile
            const int t = threadIdx.x - 64;
            for (int it = t; it < BN * 2; it += 128) {
              const int j = it % BN, hh = it / BN;
              const int m = mb + j;
              const int n0 = tile_a * BM + hh * 64;
              if (m < g.rows_b && n0 < g.rows_a) {
                float x[64];
#pragma unroll
                for (int k = 0; k < 64; ++k) x[k] = stage[j * (BM + 1) + hh * 64 + k];
                qkv_emit(e, n0 / e.attn_dim, (n0 % e.attn_dim) / 64, m, x);
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
    if (lane == 0) mbar_wait(accb, 0, g.status, kStatusTimeoutDrain, nullptr);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int BN, bool SWAP>
cudaError_t prepare_bn() {
  return cudaFuncSetAttribute(tc_gemm_kernel<BN, SWAP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              TileCfg<BN>::kSmem);
}

template <int BN, bool SWAP>
cudaError_t launch_bn(const TcGemm& t, const EpiArgs& e, cudaStream_t s) {
  using C = TileCfg<BN>;
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
  g.ws = t.ws;
  g.tickets = t.tickets;
  g.status = t.status;
  dim3 grid((t.rows_a + BM - 1) / BM, (t.rows_b + BN - 1) / BN, splits);
  tc_gemm_kernel<BN, SWAP><<<grid, kThreads, C::kSmem, s>>>(*t.map_a, *t.map_b, g, e);
  return cudaGetLastError();
}

}  // namespace

cudaError_t prepare_tc_gemm() {
  cudaError_t e;
  if ((e = prepare_bn<32, true>()) != cudaSuccess) return e;
  if ((e = prepare_bn<64, true>()) != cudaSuccess) return e;
  if ((e = prepare_bn<128, true>()) != cudaSuccess) return e;
  if ((e = prepare_bn<256, true>()) != cudaSuccess) return e;
  if ((e = prepare_bn<64, false>()) != cudaSuccess) return e;
  if ((e = prepare_bn<128, false>()) != cudaSuccess) return e;
  return prepare_bn<256, false>();
}

cudaError_t launch_tc_gemm(const TcGemm& t, const EpiArgs& e, cudaStream_t s) {
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
      case 128: return launch_bn<128, false>(t, e, s);
      case 256: return launch_bn<256, false>(t, e, s);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace wam
