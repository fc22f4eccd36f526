// fp32 SIMT GEMM with the same epilogues as the tensor-core path -- the
// debug-precision twin used by fp32 models (tolerance 1e-4 against the
// oracle).  C[m, n] = sum_k X[m, k] W[n, k]; 64 x 64 tiles, 256 threads, 4 x 4
// outputs per thread, K staged through shared memory in steps of 16.
#include "common.cuh"
#include "kernels.h"

namespace wam {
namespace {

constexpr int T = 64, TK = 16;

__device__ __forceinline__ void epi_elem_f32(const EpiArgs& e, int m, int n, float acc) {
  const float y = acc + e.bias[n];
  const size_t idx = (size_t)m * e.ld_out + n;
  switch (e.kind) {
    case kEpiStoreF32:
      e.out_f32[idx] = y;
      break;
    case kEpiGateRes:
      e.out_f32[idx] += e.gate[n] * y;
      break;
    case kEpiGelu:
      reinterpret_cast<float*>(e.out_act)[idx] = gelu_tanh(y);
      break;
    case kEpiScaleAct:
      reinterpret_cast<float*>(e.out_act)[idx] = e.scale * y;
      break;
    case kEpiEuler: {
      const float dt = e.aio->sched[e.step] - e.aio->sched[e.step + 1];
      e.out_f32[idx] -= dt * y;
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
      if (e.out_act) reinterpret_cast<float*>(e.out_act)[(size_t)m * e.a_next_ld + n] = xn;
      if (e.step == e.vio->vsteps - 1) e.vio->video_out[idx] = xn;
      break;
    }
    default:
      break;
  }
}

__global__ void __launch_bounds__(256) f32_gemm_kernel(const float* __restrict__ X, int ldx,
                                                       const float* __restrict__ W, int M, int N, int K,
                                                       const EpiArgs e) {
  __shared__ float sX[TK][T + 4];
  __shared__ float sW[TK][T + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * T, n0 = blockIdx.x * T;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += TK) {
    for (int i = threadIdx.x; i < T * TK; i += 256) {
      const int r = i / TK, c = i % TK;
      const int m = m0 + r, n = n0 + r, k = k0 + c;
      sX[c][r] = (m < M && k < K) ? X[(size_t)m * ldx + k] : 0.f;
      sW[c][r] = (n < N && k < K) ? W[(size_t)n * K + k] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < TK; ++c) {
      float xv[4], wv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        xv[i] = sX[c][ty * 4 + i];
        wv[i] = sW[c][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] += xv[i] * wv[j];
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = m0 + ty * 4 + i, n = n0 + tx * 4 + j;
      if (m < M && n < N) epi_elem_f32(e, m, n, acc[i][j]);
    }
}

// QK-RMSNorm (gain) + RoPE + scatter for the fp32 path; one thread per
// (token, section, head) of the raw projection qkv [M, 3A] (bias included).
__global__ void qkv_post_f32_kernel(const float* __restrict__ qkv, int M, const EpiArgs e) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  const int H = e.n_heads, Dh = e.head_dim, A = e.attn_dim;
  if (idx >= M * 3 * H) return;
  const int head = idx % H, section = (idx / H) % 3, m = idx / (3 * H);
  const int b = m / e.seq_len, l = m - b * e.seq_len;
  float x[128];
  const float* src = qkv + (size_t)m * 3 * A + section * A + head * Dh;
  for (int j = 0; j < Dh; ++j) x[j] = src[j];
  if (section < 2) {
    const float* g = (section == 0 ? e.gq : e.gk) + head * Dh;
    float ss = 0.f;
    for (int j = 0; j < Dh; ++j) ss += x[j] * x[j];
    const float r = 1.0f / sqrtf(ss / (float)Dh + 1e-6f);
    for (int j = 0; j < Dh; ++j) x[j] *= r * g[j];
    const int half = Dh / 2, pos = e.cache_off + l;
    for (int j = 0; j < half; ++j) {
      const float c = e.rope_cos[pos * half + j], s = e.rope_sin[pos * half + j];
      const float x1 = x[j], x2 = x[j + half];
      x[j] = x1 * c - x2 * s;
      x[j + half] = x1 * s + x2 * c;
    }
  }
  float* dst;
  if (section == 0)
    dst = reinterpret_cast<float*>(e.q_out) + ((size_t)(b * H + head) * e.seq_len + l) * Dh;
  else
    dst = reinterpret_cast<float*>(section == 1 ? e.k_cache : e.v_cache) +
          ((size_t)(b * H + head) * e.cache_len + e.cache_off + l) * Dh;
  for (int j = 0; j < Dh; ++j) dst[j] = x[j];
}

}  // namespace

cudaError_t launch_f32_gemm(const float* X, int ldx, const float* W, int M, int N, int K, const EpiArgs& e,
                            cudaStream_t s) {
  dim3 grid((N + T - 1) / T, (M + T - 1) / T);
  f32_gemm_kernel<<<grid, 256, 0, s>>>(X, ldx, W, M, N, K, e);
  return cudaGetLastError();
}

cudaError_t launch_qkv_post_f32(const float* qkv, int M, const EpiArgs& e, cudaStream_t s) {
  if (e.head_dim > 128) return cudaErrorInvalidValue;
  const int n = M * 3 * e.n_heads;
  qkv_post_f32_kernel<<<(n + 127) / 128, 128, 0, s>>>(qkv, M, e);
  return cudaGetLastError();
}

}  // namespace wam
