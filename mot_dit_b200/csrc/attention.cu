// Attention of the MoT blocks.
//
// Video queries attend over the video keys of their block; action queries
// attend over the concatenation [K^v_i; K^a_i] / [V^v_i; V^a_i] (RealtimeWAM
// summary page, 前置知识 "Mixture-of-Transformers" and "KV 缓存").  Both read
// the per-block cache [B, H, L_v + L_a, Dh]: rows [0, L_v) are the video
// expert's K/V, rows [L_v, L_v + L_a) the action expert's, so the joint key
// list is one contiguous row range and the video attention simply stops at L_v.
//
// bf16 path: flash-attention over 64-key tiles with mma.sync m16n8k16 (bf16
// in, fp32 accumulate), online softmax in fp32, P rounded to bf16 for the PV
// product.  The video attention is one pass per 64-query tile.  The action
// attention (32 queries, ~1.1k keys, bound by reading the video K/V) splits
// the key range over CTAs; each writes an unnormalised partial (O, row max,
// row sum) and the last CTA of a (sample, head) -- found with an integer
// ticket -- combines the partials in split order, so the result does not
// depend on CTA timing.
//
// fp32 path: one warp per (query, head), exact fp32 softmax (debug precision).
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace wam {
WAM_KTRACE_UNIT(jattn)
namespace {

constexpr int kD = 64;      // head dim of the bf16 path
constexpr int kTQ = 64;     // queries per CTA (4 warps x 16)
constexpr int kTK = 64;     // keys per tile
constexpr int kAttnThreads = 128;
constexpr int kMaxSplits = 32;  // key splits of the action attention
constexpr int kCombineBytes = 96 * 1024;  // dynamic shared memory for staging partial O rows
constexpr int kJMaxSplits = 8;  // joint action attention: CTAs per cluster (key splits)

// Row-major [64][64] bf16 tile, 16-byte chunks XOR-swizzled by row.
__device__ __forceinline__ uint32_t tile_off(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void load_tile(uint32_t s_base, const __nv_bfloat16* g, int row0, int rows_valid,
                                          int tid) {
  // 64 rows x 8 chunks of 16 bytes
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int idx = tid + i * kAttnThreads;
    const int r = idx >> 3, c = idx & 7;
    const bool ok = (row0 + r) < rows_valid;
    const __nv_bfloat16* src = g + (size_t)(ok ? row0 + r : 0) * kD + c * 8;
    cp_async16(s_base + tile_off(r, c), src, ok);
  }
}

template <bool SPLIT>
__global__ void __launch_bounds__(kAttnThreads)
    attn_bf16_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kc,
                     const __nv_bfloat16* __restrict__ vc, __nv_bfloat16* __restrict__ out, int H, int Lq,
                     int Lk, int Lcache, int splits, int keys_per_split, float* __restrict__ ws,
                     int* __restrict__ tickets, int rows_per_pass, int ldo) {
  __shared__ __align__(128) uint8_t smem[kTQ * 128 + 2 * 2 * kTK * 128];
  extern __shared__ float4 s_comb[];  // split path: [splits][rows_per_pass][16] partial O rows
  __shared__ int s_last;
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sK0 = sQ + kTQ * 128;
  const uint32_t sV0 = sK0 + 2 * kTK * 128;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const int h = blockIdx.y;
  const int b = blockIdx.z / splits, split = blockIdx.z % splits;
  const int q0 = blockIdx.x * kTQ;
  const int k_begin = split * keys_per_split;
  const int k_end = min(Lk, k_begin + keys_per_split);
  const int ntiles = (k_end - k_begin + kTK - 1) / kTK;

  pdl_trigger();
  pdl_wait();
  const __nv_bfloat16* qb = q + (size_t)(b * H + h) * Lq * kD;
  const __nv_bfloat16* kb = kc + (size_t)(b * H + h) * Lcache * kD;
  const __nv_bfloat16* vb = vc + (size_t)(b * H + h) * Lcache * kD;

  load_tile(sQ, qb, q0, Lq, tid);
  load_tile(sK0, kb, k_begin, k_end, tid);
  load_tile(sV0, vb, k_begin, k_end, tid);
  cp_async_commit();

  const float sl2e = 1.4426950408889634f * rsqrtf((float)kD);
  float o[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  uint32_t qf[4][4];

  for (int t = 0; t < ntiles; ++t) {
    const int buf = t & 1;
    if (t + 1 < ntiles) {
      const int nb = (t + 1) & 1;
      load_tile(sK0 + nb * kTK * 128, kb, k_begin + (t + 1) * kTK, k_end, tid);
      load_tile(sV0 + nb * kTK * 128, vb, k_begin + (t + 1) * kTK, k_end, tid);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (t == 0) {
#pragma unroll
      for (int kt = 0; kt < 4; ++kt) {
        const int r = warp * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int c = kt * 2 + (lane >> 4);
        ldsm_x4(sQ + tile_off(r, c), qf[kt][0], qf[kt][1], qf[kt][2], qf[kt][3]);
      }
    }
    const uint32_t sK = sK0 + buf * kTK * 128, sV = sV0 + buf * kTK * 128;
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kt = 0; kt < 4; ++kt) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const int r = np * 16 + (lane & 7) + 8 * (lane >> 4);
        const int c = kt * 2 + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sK + tile_off(r, c), b0, b1, b2, b3);
        mma_bf16_16816(s[2 * np], qf[kt][0], qf[kt][1], qf[kt][2], qf[kt][3], b0, b1);
        mma_bf16_16816(s[2 * np + 1], qf[kt][0], qf[kt][1], qf[kt][2], qf[kt][3], b2, b3);
      }
    }
    // mask keys past the end of this split / of the key list
    const int kbase = k_begin + t * kTK;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int k0 = kbase + nt * 8 + 2 * t4;
      if (k0 >= k_end) s[nt][0] = s[nt][2] = -INFINITY;
      if (k0 + 1 >= k_end) s[nt][1] = s[nt][3] = -INFINITY;
    }
    // online softmax, rows g (r = 0) and g + 8 (r = 1)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) mx = fmaxf(mx, fmaxf(s[nt][2 * r], s[nt][2 * r + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_run[r], mx);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = exp2f((m_run[r] - m_use) * sl2e);
      float rs = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const float p0 = exp2f((s[nt][2 * r] - m_use) * sl2e);
        const float p1 = exp2f((s[nt][2 * r + 1] - m_use) * sl2e);
        s[nt][2 * r] = p0;
        s[nt][2 * r + 1] = p1;
        rs += p0 + p1;
      }
      l_run[r] = l_run[r] * alpha + rs;
      m_run[r] = m_new;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        o[nt][2 * r] *= alpha;
        o[nt][2 * r + 1] *= alpha;
      }
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint32_t a0 = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      const uint32_t a1 = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      const uint32_t a2 = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      const uint32_t a3 = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int dp = 0; dp < 4; ++dp) {
        const int r = kk * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int c = dp * 2 + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sV + tile_off(r, c), b0, b1, b2, b3);
        mma_bf16_16816(o[2 * dp], a0, a1, a2, a3, b0, b1);
        mma_bf16_16816(o[2 * dp + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    __syncthreads();
  }

  float l_tot[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    float l = l_run[r];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    l_tot[r] = l;
  }
  const int A = ldo;  // row stride of out
  if (!SPLIT) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int qi = q0 + warp * 16 + g + 8 * r;
      if (qi < Lq) {
        const float inv = 1.0f / l_tot[r];
        __nv_bfloat16* dst = out + (size_t)(b * Lq + qi) * A + h * kD;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
          *reinterpret_cast<uint32_t*>(dst + nt * 8 + 2 * t4) =
              pack_bf16(o[nt][2 * r] * inv, o[nt][2 * r + 1] * inv);
      }
    }
    return;
  }
  // ---- split: partials to the workspace, last CTA of (b, h) combines
  const size_t bh = (size_t)b * H + h;
  float* wO = ws + (bh * splits + split) * (kTQ * kD);
  float* wM = ws + (size_t)gridDim.z / splits * H * splits * kTQ * kD + (bh * splits + split) * kTQ * 2;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = warp * 16 + g + 8 * r;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
      *reinterpret_cast<float2*>(wO + row * kD + nt * 8 + 2 * t4) = make_float2(o[nt][2 * r], o[nt][2 * r + 1]);
    if (t4 == 0) {
      wM[row * 2] = m_run[r];
      wM[row * 2 + 1] = l_tot[r];
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(tickets + bh, 1) == splits - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // Combine in split order: per row r, M = max_s m_s, den = sum_s 2^((m_s - M) c) l_s,
  // then O[r, :] = sum_s (2^((m_s - M) c) / den) O_s[r, :].
  // the Q/K/V tiles are no longer needed: reuse them for the per-row factors
  float (*s_f)[kTQ] = reinterpret_cast<float (*)[kTQ]>(smem);
  const float* cO = ws + bh * splits * (kTQ * kD);
  const float* cM = ws + (size_t)gridDim.z / splits * H * splits * kTQ * kD + bh * splits * kTQ * 2;
  // every (m, l) of every split in flight at once, into shared memory
  float* s_ml = reinterpret_cast<float*>(smem) + kMaxSplits * kTQ;  // [splits][kTQ][2]
  for (int i = tid; i < splits * kTQ * 2; i += kAttnThreads) s_ml[i] = __ldcg(cM + i);
  __syncthreads();
  if (tid < kTQ) {
    float M = -INFINITY;
    for (int s2 = 0; s2 < splits; ++s2) M = fmaxf(M, s_ml[(s2 * kTQ + tid) * 2]);
    float den = 0.f;
    for (int s2 = 0; s2 < splits; ++s2) {
      const float f = exp2f((s_ml[(s2 * kTQ + tid) * 2] - M) * sl2e);
      s_f[s2][tid] = f;
      den += f * s_ml[(s2 * kTQ + tid) * 2 + 1];
    }
    const float inv = 1.0f / den;
    for (int s2 = 0; s2 < splits; ++s2) s_f[s2][tid] *= inv;
  }
  __syncthreads();
  // Stage the partial O rows of every split in shared memory, all copies in
  // flight at once (the reads are L2-latency bound otherwise), then sum them
  // in split order.
  for (int r0 = 0; r0 < Lq; r0 += rows_per_pass) {
    const int nr = min(rows_per_pass, Lq - r0);
    for (int i = tid; i < splits * nr * 16; i += kAttnThreads) {
      const int s2 = i / (nr * 16), rem = i - s2 * (nr * 16);
      const int row = rem >> 4, c4 = rem & 15;
      cp_async16(smem_u32(s_comb + (s2 * nr + row) * 16 + c4), cO + (size_t)s2 * kTQ * kD + (r0 + row) * kD + 4 * c4,
                 true);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    for (int i = tid; i < nr * 16; i += kAttnThreads) {
      const int row = i >> 4, c4 = i & 15;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s2 = 0; s2 < splits; ++s2) {
        const float f = s_f[s2][r0 + row];
        const float4 v4 = s_comb[(s2 * nr + row) * 16 + c4];
        acc.x += f * v4.x;
        acc.y += f * v4.y;
        acc.z += f * v4.z;
        acc.w += f * v4.w;
      }
      uint2 w;
      w.x = pack_bf16(acc.x, acc.y);
      w.y = pack_bf16(acc.z, acc.w);
      *reinterpret_cast<uint2*>(out + (size_t)(b * Lq + r0 + row) * A + h * kD + 4 * c4) = w;
    }
    __syncthreads();
  }
  if (tid == 0) tickets[bh] = 0;
}

// fp32 debug attention: one warp per (query, head, sample).
template <int D>
__global__ void attn_f32_kernel(const float* __restrict__ q, const float* __restrict__ kc,
                                const float* __restrict__ vc, float* __restrict__ out, int H, int Lq, int Lk,
                                int Lcache, int total, int ldo) {
  const int warp_global = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (warp_global >= total) return;  // uniform per warp
  const int lane = threadIdx.x & 31;
  const int qi = warp_global % Lq;
  const int h = (warp_global / Lq) % H;
  const int b = warp_global / (Lq * H);
  const float* qr = q + ((size_t)(b * H + h) * Lq + qi) * D;
  const float* kb = kc + (size_t)(b * H + h) * Lcache * D;
  const float* vb = vc + (size_t)(b * H + h) * Lcache * D;
  const float scale = 1.0f / sqrtf((float)D);
  float qv[D];
#pragma unroll
  for (int d = 0; d < D; ++d) qv[d] = qr[d];
  float m = -INFINITY, l = 0.f, acc[D];
#pragma unroll
  for (int d = 0; d < D; ++d) acc[d] = 0.f;
  for (int k = lane; k < Lk; k += 32) {
    float s = 0.f;
#pragma unroll
    for (int d = 0; d < D; ++d) s += qv[d] * kb[(size_t)k * D + d];
    s *= scale;
    const float m_new = fmaxf(m, s);
    const float alpha = expf(m - m_new);
    const float p = expf(s - m_new);
    l = l * alpha + p;
#pragma unroll
    for (int d = 0; d < D; ++d) acc[d] = acc[d] * alpha + p * vb[(size_t)k * D + d];
    m = m_new;
  }
  float M = m;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float f = (m == -INFINITY) ? 0.f : expf(m - M);
  l *= f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  float* dst = out + (size_t)(b * Lq + qi) * ldo + h * D;
#pragma unroll
  for (int d = 0; d < D; ++d) {
    float v = acc[d] * f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) dst[d] = v / l;
  }
}

// ------------------------------------------------ joint action attention --
// The action queries of one (sample, head) against the joint key list, split
// over the `splits` CTAs of a cluster (rank = split): each takes keys
// [split * kps, (split + 1) * kps) in 64-key tiles, brought in by TMA into a
// kJStages-deep mbarrier ring.  Tiles of cache rows below `ready` (rows the
// caller guarantees complete at launch) are requested before the
// dependent-launch wait, while the previous kernel still runs; the chunk
// passes 0 (a captured cross-stream event edge is programmatic too, so the
// video rows are complete only after the wait).  Flash loop as above
// (mma.sync, online softmax in fp32); each CTA then stores its unnormalised
// partial (O, row max, row sum) into rank 0's shared memory through the
// cluster's shared window, and rank 0 merges them in split order, so the
// result does not depend on timing.
constexpr int kJStages = 4;
constexpr int kJThreads = 128;
constexpr int kKVTile = kTK * kD * 2;  // 8 KB: one K or V tile (64 rows x 128 B)

struct AttnJointK {
  int H, Lq, Lk, splits, kps, ready, ld_out;
  const int* ready_flag;  // non-null: `ready` applies only if it reads 1
  int zk0, zv0;
  const __nv_bfloat16* q;
  __nv_bfloat16* out;
  unsigned* status;
};

__device__ __forceinline__ void jt_cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t jt_cluster_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_cluster_f2(uint32_t addr, float x, float y) {
  asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(x), "f"(y) : "memory");
}

// The K/V ring and the Q tile; after the flash loop rank 0's copy of this
// region holds the partials ([split][Lq][64] O, then [split][Lq][2] max / sum).
constexpr int kJRegion = kJStages * 2 * kKVTile + kTQ * 128;
constexpr size_t kJSmem = kJRegion + kJStages * 8;
// A launch that has the GPU to itself asks for more than it needs, so that its
// CTAs land one per SM (each with the SM's whole L1 / TMA bandwidth): the
// 10-step chunk ran 19.07 ms this way against 19.77 ms at three per SM.
constexpr size_t kJSmemSpread = 120 * 1024;
// Splits whose partials fit the region: splits * Lq * (64 + 2) floats.
__host__ __device__ constexpr bool joint_fits(int splits, int Lq) { return (size_t)splits * Lq * (kD + 2) * 4 <= kJRegion; }

__global__ void __launch_bounds__(kJThreads, 1)
    attn_joint_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                      const AttnJointK a) {
  WAM_KT_BEGIN;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // TMA's 128-byte swizzle is a function of the address bits (tile bases on
  // 1024-byte boundaries); every CTA of the cluster sees the same layout
  if (smem_u32(smem_raw) & 1023) {
    if (threadIdx.x == 0) atomicOr(a.status, kStatusTimeoutDrain);
    return;
  }
  uint8_t* sKV = smem_raw;                                   // [stage][K | V]
  uint8_t* sQ = sKV + kJStages * 2 * kKVTile;                // [64][128 B]
  float* sO = reinterpret_cast<float*>(smem_raw);            // rank 0, after the loop: [split][Lq][64] partial O
  float* sML = sO + a.splits * a.Lq * kD;                    // rank 0, after the loop: [split][Lq][2] max, sum
  uint64_t* full = reinterpret_cast<uint64_t*>(smem_raw + kJRegion);
  __shared__ int s_abort;
  __shared__ float s_f[kJMaxSplits * kTQ];  // rank 0: merge weights [split][row]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const int split = blockIdx.x % a.splits;  // = the rank in the cluster
  const int bh = blockIdx.x / a.splits;
  const int b = bh / a.H, h = bh % a.H;
  const int k_begin = split * a.kps;
  const int k_end = min(a.Lk, k_begin + a.kps);
  const int ntiles = k_end > k_begin ? (k_end - k_begin + kTK - 1) / kTK : 0;

  if (tid == 0) {
    for (int st = 0; st < kJStages; ++st) mbar_init(&full[st], 1);
    s_abort = 0;
    fence_barrier_init();
    prefetch_tensormap(&map_k);
    prefetch_tensormap(&map_v);
  }
  __syncthreads();
  pdl_trigger();

  auto issue = [&](int t) {  // tile t into stage t % kJStages
    const int st = t % kJStages;
    mbar_arrive_expect_tx(&full[st], 2 * kKVTile);
    tma_load_3d(sKV + st * 2 * kKVTile, &map_k, &full[st], 0, k_begin + t * kTK, a.zk0 + bh);
    tma_load_3d(sKV + st * 2 * kKVTile + kKVTile, &map_v, &full[st], 0, k_begin + t * kTK, a.zv0 + bh);
  };
  const int first = min(ntiles, kJStages);
  int issued = 0;
  if (tid == 0) {  // tiles of keys complete before the launch
    int ready = a.ready;
    if (a.ready_flag) {
      int f;
      asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(f) : "l"(a.ready_flag) : "memory");
      if (f != 1) ready = 0;
      else  // the rows were written before the flag was set; TMA (the async proxy) reads them next
        asm volatile("fence.proxy.async.global;" ::: "memory");
    }
    while (issued < first && min(k_end, k_begin + (issued + 1) * kTK) <= ready) issue(issued++);
  }
  pdl_wait();  // the queries and the action rows are the previous kernel's
  WAM_KT_WAITED();
  if (tid == 0)
    while (issued < first) issue(issued++);
  const __nv_bfloat16* qb = a.q + (size_t)bh * a.Lq * kD;
  load_tile(smem_u32(sQ), qb, 0, a.Lq, tid);
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  const float sl2e = 1.4426950408889634f * rsqrtf((float)kD);
  float o[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  // Up to 32 queries: warp w takes query rows 16 (w & 1) .. + 15 and the key
  // tiles of parity w >> 1, so two warp pairs work on two tiles at once and
  // merge at the end; up to 64 queries: warp w takes rows 16 w .. + 15 and
  // every tile.
  const bool halves = a.Lq <= 32;
  const int tpi = halves ? 2 : 1;  // tiles per iteration
  const int qrow0 = (halves ? (warp & 1) : warp) * 16;
  const int kh = halves ? (warp >> 1) : 0;
  uint32_t qf[4][4];
#pragma unroll
  for (int kt = 0; kt < 4; ++kt) {
    const int r = qrow0 + (lane & 7) + 8 * ((lane >> 3) & 1);
    const int c = kt * 2 + (lane >> 4);
    ldsm_x4(smem_u32(sQ) + tile_off(r, c), qf[kt][0], qf[kt][1], qf[kt][2], qf[kt][3]);
  }

  int consumed = 0;  // (thread 0) tiles whose copies have landed
  for (int t0 = 0; t0 < ntiles; t0 += tpi) {
    if (tid == 0) {
      for (int u = t0; u < min(ntiles, t0 + tpi); ++u) {
        if (mbar_wait(&full[u % kJStages], (u / kJStages) & 1, a.status, kStatusTimeoutTmaFull, nullptr)) {
          consumed = u + 1;
        } else {
          s_abort = 1;
          break;
        }
      }
    }
    __syncthreads();
    if (s_abort) break;  // (uniform: read after the barrier)
    const int t = t0 + kh;
    if (t >= ntiles) {  // (the odd pair past the last tile)
      __syncthreads();
      continue;
    }
    const int st = t % kJStages;
    const uint32_t sK = smem_u32(sKV + st * 2 * kKVTile), sV = sK + kKVTile;
    float s_[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s_[i][0] = s_[i][1] = s_[i][2] = s_[i][3] = 0.f;
#pragma unroll
    for (int kt = 0; kt < 4; ++kt) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const int r = np * 16 + (lane & 7) + 8 * (lane >> 4);
        const int c = kt * 2 + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sK + tile_off(r, c), b0, b1, b2, b3);
        mma_bf16_16816(s_[2 * np], qf[kt][0], qf[kt][1], qf[kt][2], qf[kt][3], b0, b1);
        mma_bf16_16816(s_[2 * np + 1], qf[kt][0], qf[kt][1], qf[kt][2], qf[kt][3], b2, b3);
      }
    }
    // keys past this split's end (the tile's tail rows belong to the next split or lie past the list)
    const int kbase = k_begin + t * kTK;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int k0 = kbase + nt * 8 + 2 * t4;
      if (k0 >= k_end) s_[nt][0] = s_[nt][2] = -INFINITY;
      if (k0 + 1 >= k_end) s_[nt][1] = s_[nt][3] = -INFINITY;
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) mx = fmaxf(mx, fmaxf(s_[nt][2 * r], s_[nt][2 * r + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_run[r], mx);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = exp2f((m_run[r] - m_use) * sl2e);
      float rs = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const float p0 = exp2f((s_[nt][2 * r] - m_use) * sl2e);
        const float p1 = exp2f((s_[nt][2 * r + 1] - m_use) * sl2e);
        s_[nt][2 * r] = p0;
        s_[nt][2 * r + 1] = p1;
        rs += p0 + p1;
      }
      l_run[r] = l_run[r] * alpha + rs;
      m_run[r] = m_new;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        o[nt][2 * r] *= alpha;
        o[nt][2 * r + 1] *= alpha;
      }
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint32_t a0 = pack_bf16(s_[2 * kk][0], s_[2 * kk][1]);
      const uint32_t a1 = pack_bf16(s_[2 * kk][2], s_[2 * kk][3]);
      const uint32_t a2 = pack_bf16(s_[2 * kk + 1][0], s_[2 * kk + 1][1]);
      const uint32_t a3 = pack_bf16(s_[2 * kk + 1][2], s_[2 * kk + 1][3]);
#pragma unroll
      for (int dp = 0; dp < 4; ++dp) {
        const int r = kk * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int c = dp * 2 + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sV + tile_off(r, c), b0, b1, b2, b3);
        mma_bf16_16816(o[2 * dp], a0, a1, a2, a3, b0, b1);
        mma_bf16_16816(o[2 * dp + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    __syncthreads();  // the stages are read
    if (tid == 0)  // tiles t0 + kJStages .. into the freed stages
      while (issued < ntiles && issued < t0 + tpi + kJStages) issue(issued++);
  }
  // never leave with copies in flight into this CTA's shared memory
  if (tid == 0)
    for (int t = consumed; t < issued; ++t)
      mbar_wait(&full[t % kJStages], (t / kJStages) & 1, a.status, kStatusTimeoutDrain, nullptr);

  float l_tot[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    float l = l_run[r];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    l_tot[r] = l;
  }
  __syncthreads();  // (thread 0's drain above: the ring is idle)
  if (halves) {
    // the odd-tile pair hands (O, m, l) over in the idle ring; the even-tile
    // pair merges them into its own (log-sum-exp weights)
    float* xo = reinterpret_cast<float*>(sKV);  // [32 rows][64]
    float* xml = xo + 32 * kD;                  // [32 rows][2]
    if (kh == 1) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int row = qrow0 + g + 8 * r;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
          *reinterpret_cast<float2*>(xo + row * kD + nt * 8 + 2 * t4) = make_float2(o[nt][2 * r], o[nt][2 * r + 1]);
        if (t4 == 0) *reinterpret_cast<float2*>(xml + row * 2) = make_float2(m_run[r], l_tot[r]);
      }
    }
    __syncthreads();
    if (kh == 0) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int row = qrow0 + g + 8 * r;
        const float2 ml1 = *reinterpret_cast<const float2*>(xml + row * 2);
        const float M = fmaxf(m_run[r], ml1.x);  // m_run[r] is finite: the even pair has tile 0
        const float f0 = exp2f((m_run[r] - M) * sl2e), f1 = exp2f((ml1.x - M) * sl2e);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          const float2 o1 = *reinterpret_cast<const float2*>(xo + row * kD + nt * 8 + 2 * t4);
          o[nt][2 * r] = o[nt][2 * r] * f0 + o1.x * f1;
          o[nt][2 * r + 1] = o[nt][2 * r + 1] * f0 + o1.y * f1;
        }
        l_tot[r] = l_tot[r] * f0 + ml1.y * f1;
        m_run[r] = M;
      }
    }
  }
  const bool owner = kh == 0;  // this warp holds merged rows
  if (a.splits == 1) {
#pragma unroll
    for (int r = 0; r < 2 && owner; ++r) {
      const int qi = qrow0 + g + 8 * r;
      if (qi < a.Lq) {
        const float inv = 1.0f / l_tot[r];
        __nv_bfloat16* dst = a.out + (size_t)(b * a.Lq + qi) * a.ld_out + h * kD;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
          *reinterpret_cast<uint32_t*>(dst + nt * 8 + 2 * t4) = pack_bf16(o[nt][2 * r] * inv, o[nt][2 * r + 1] * inv);
      }
    }
    WAM_KT_END(jattn, 3u);
    return;
  }
  // partial of this split -> rank 0's shared memory, once every CTA of the
  // cluster is done with its ring (rank 0's is overwritten)
  jt_cluster_sync();
  const uint32_t rO = jt_cluster_addr(sO + (size_t)split * a.Lq * kD, 0);
  const uint32_t rML = jt_cluster_addr(sML + (size_t)split * a.Lq * 2, 0);
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = qrow0 + g + 8 * r;
    if (owner && row < a.Lq) {
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
        st_cluster_f2(rO + (uint32_t)(row * kD + nt * 8 + 2 * t4) * 4, o[nt][2 * r], o[nt][2 * r + 1]);
      if (t4 == 0) st_cluster_f2(rML + (uint32_t)row * 8, m_run[r], l_tot[r]);
    }
  }
  jt_cluster_sync();  // every partial is in rank 0's shared memory
  if (split != 0) {
    WAM_KT_END(jattn, 3u);
    return;
  }
  // merge in split order: M = max_s m_s, f_s = 2^((m_s - M) c) / sum_s 2^((m_s - M) c) l_s
  if (tid < a.Lq) {
    float M = -INFINITY;
    for (int s2 = 0; s2 < a.splits; ++s2) M = fmaxf(M, sML[(s2 * a.Lq + tid) * 2]);
    float den = 0.f;
    for (int s2 = 0; s2 < a.splits; ++s2) {
      const float f = exp2f((sML[(s2 * a.Lq + tid) * 2] - M) * sl2e);
      s_f[s2 * kTQ + tid] = f;
      den += f * sML[(s2 * a.Lq + tid) * 2 + 1];
    }
    const float inv = 1.0f / den;
    for (int s2 = 0; s2 < a.splits; ++s2) s_f[s2 * kTQ + tid] *= inv;
  }
  __syncthreads();
  for (int i = tid; i < a.Lq * (kD / 4); i += kJThreads) {
    const int row = i / (kD / 4), c4 = i % (kD / 4);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s2 = 0; s2 < a.splits; ++s2) {
      const float f = s_f[s2 * kTQ + row];
      const float4 v4 = reinterpret_cast<const float4*>(sO + ((size_t)s2 * a.Lq + row) * kD)[c4];
      acc.x += f * v4.x;
      acc.y += f * v4.y;
      acc.z += f * v4.z;
      acc.w += f * v4.w;
    }
    uint2 w;
    w.x = pack_bf16(acc.x, acc.y);
    w.y = pack_bf16(acc.z, acc.w);
    *reinterpret_cast<uint2*>(a.out + (size_t)(b * a.Lq + row) * a.ld_out + h * kD + 4 * c4) = w;
  }
  WAM_KT_END(jattn, 3u);
}

}  // namespace

size_t attention_ws_floats(int B, int H, int Dh, int Lq, int splits) {
  (void)Dh;
  (void)Lq;
  return (size_t)B * H * splits * (kTQ * kD + kTQ * 2);
}

cudaError_t prepare_attention_bf16() {
  return cudaFuncSetAttribute(attn_bf16_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kCombineBytes);
}

cudaError_t launch_attention_bf16(const AttnArgs& a, cudaStream_t s) {
  if (a.Dh != kD) return cudaErrorInvalidValue;
  const int ldo = a.ld_out ? a.ld_out : a.H * kD;
  if (ldo < a.H * kD || ldo % 4) return cudaErrorInvalidValue;
  const int splits = a.splits < 1 ? 1 : a.splits;
  if (splits > 1 && a.Lq > kTQ) return cudaErrorInvalidValue;
  int kps = (a.Lk + splits - 1) / splits;
  kps = (kps + kTK - 1) / kTK * kTK;
  const int used = (a.Lk + kps - 1) / kps;  // non-empty splits only
  if (used > kMaxSplits) return cudaErrorInvalidValue;
  dim3 grid((a.Lq + kTQ - 1) / kTQ, a.H, a.B * used);
  const auto* q = reinterpret_cast<const __nv_bfloat16*>(a.q);
  const auto* k = reinterpret_cast<const __nv_bfloat16*>(a.k);
  const auto* v = reinterpret_cast<const __nv_bfloat16*>(a.v);
  auto* o = reinterpret_cast<__nv_bfloat16*>(a.out);
  if (used > 1) {
    const int rpp = std::max(1, std::min(a.Lq, kCombineBytes / (used * kD * 4)));
    return launch_k(attn_bf16_kernel<true>, grid, dim3(kAttnThreads), (size_t)used * rpp * kD * 4, s, q, k, v, o,
                    a.H, a.Lq, a.Lk, a.Lcache, used, kps, a.ws, a.tickets, rpp, ldo);
  }
  return launch_k(attn_bf16_kernel<false>, grid, dim3(kAttnThreads), 0, s, q, k, v, o, a.H, a.Lq, a.Lk, a.Lcache, 1,
                  kps, (float*)nullptr, (int*)nullptr, 0, ldo);
}

cudaError_t launch_attention_f32(const AttnArgs& a, cudaStream_t s) {
  const int ldo = a.ld_out ? a.ld_out : a.H * a.Dh;
  if (ldo < a.H * a.Dh) return cudaErrorInvalidValue;
  const int warps = a.B * a.H * a.Lq;
  const int per_block = 4;
  dim3 grid((warps + per_block - 1) / per_block);
  const auto* q = reinterpret_cast<const float*>(a.q);
  const auto* k = reinterpret_cast<const float*>(a.k);
  const auto* v = reinterpret_cast<const float*>(a.v);
  auto* o = reinterpret_cast<float*>(a.out);
  switch (a.Dh) {
    case 16: attn_f32_kernel<16><<<grid, 32 * per_block, 0, s>>>(q, k, v, o, a.H, a.Lq, a.Lk, a.Lcache, warps, ldo); break;
    case 32: attn_f32_kernel<32><<<grid, 32 * per_block, 0, s>>>(q, k, v, o, a.H, a.Lq, a.Lk, a.Lcache, warps, ldo); break;
    case 64: attn_f32_kernel<64><<<grid, 32 * per_block, 0, s>>>(q, k, v, o, a.H, a.Lq, a.Lk, a.Lcache, warps, ldo); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

int attention_joint_splits(int BH, int Lq, int Lk, int num_sms) {
  int sp = 1;
  while (sp < kJMaxSplits && BH * sp * 2 <= num_sms && Lk >= 2 * sp * kTK && joint_fits(2 * sp, Lq)) sp *= 2;
  return sp;
}

cudaError_t prepare_attention_joint() {
  return cudaFuncSetAttribute(attn_joint_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kJSmemSpread);
}

cudaError_t launch_attention_joint(const AttnJoint& t, cudaStream_t s) {
  const int ldo = t.ld_out ? t.ld_out : t.H * kD;
  if (t.Lq < 1 || t.Lq > kTQ || t.Lk < 1 || t.B < 1 || t.H < 1 || ldo < t.H * kD || ldo % 4) return cudaErrorInvalidValue;
  if (t.splits != 1 && t.splits != 2 && t.splits != 4 && t.splits != 8) return cudaErrorInvalidValue;
  if (!joint_fits(t.splits, t.Lq)) return cudaErrorInvalidValue;
  AttnJointK k;
  k.H = t.H;
  k.Lq = t.Lq;
  k.Lk = t.Lk;
  k.splits = t.splits;
  k.kps = (t.Lk + t.splits - 1) / t.splits;
  k.ready = t.ready;
  k.ready_flag = t.ready_flag;
  k.ld_out = ldo;
  k.zk0 = t.zk0;
  k.zv0 = t.zv0;
  k.q = reinterpret_cast<const __nv_bfloat16*>(t.q);
  k.out = reinterpret_cast<__nv_bfloat16*>(t.out);
  k.status = t.status;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(t.B * t.H * t.splits);
  cfg.blockDim = dim3(kJThreads);
  cfg.dynamicSmemBytes = t.spread ? kJSmemSpread : kJSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeClusterDimension;
  attr[na].val.clusterDim.x = t.splits;
  attr[na].val.clusterDim.y = 1;
  attr[na].val.clusterDim.z = 1;
  ++na;
  if (pdl_enabled()) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, attn_joint_kernel, *t.map_k, *t.map_v, k);
}

}  // namespace wam
