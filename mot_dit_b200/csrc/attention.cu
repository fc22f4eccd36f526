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
namespace {

constexpr int kD = 64;      // head dim of the bf16 path
constexpr int kTQ = 64;     // queries per CTA (4 warps x 16)
constexpr int kTK = 64;     // keys per tile
constexpr int kAttnThreads = 128;
constexpr int kMaxSplits = 32;  // key splits of the action attention
constexpr int kCombineBytes = 96 * 1024;  // dynamic shared memory for staging partial O rows

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

}  // namespace wam
