// Device pieces of the TACD target forward (Teacher-Anchored Consistency
// Distillation; RealtimeWAM summary page, 前置知识 "一致性蒸馏", 核心方法 and
// 方法步骤详情): the noising of the clean action chunk, and the targets and
// losses formed from the teacher, student and EMA results.  The networks
// themselves run on the chunk path (the video expert once, the action
// expert's Euler steps); these kernels only combine their outputs.
#include "common.cuh"
#include "kernels.h"

namespace wam {
namespace {

constexpr int kTacdThreads = 256;

// a_t = (1 - t) a_0 + t eps (the flow-matching interpolation, 方法步骤详情).
__global__ void tacd_noise_kernel(const float* __restrict__ a_clean, const float* __restrict__ eps, float t,
                                  float* __restrict__ a_t, int n) {
  pdl_trigger();
  pdl_wait();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    a_t[i] = (1.0f - t) * a_clean[i] + t * eps[i];
}

// u_TA = (a_t - a_0^T) / t, v_student = (a_t - f_student) / t,
// u_CD = (a_t - f_EMA) / t, and per sample ||v_student - u_TA||^2,
// ||v_student - u_CD||^2 over its [L_a, P_a] chunk, averaged over the batch:
// losses[0] = L_TA, losses[1] = L_CD, losses[2] = L_CD + lambda L_TA.
// One CTA; every sum runs in a fixed order (strided per thread, then a fixed
// tree), so the losses do not depend on timing.
__global__ void __launch_bounds__(kTacdThreads)
    tacd_targets_kernel(const float* __restrict__ a_t, const float* __restrict__ a0_teacher,
                        const float* __restrict__ f_student, const float* __restrict__ f_ema, float t, float lambda,
                        int B, int per_sample, float* __restrict__ u_ta, float* __restrict__ v_student,
                        float* __restrict__ u_cd, float* __restrict__ losses) {
  __shared__ float red[2][kTacdThreads];
  pdl_trigger();
  pdl_wait();
  const float inv_t = 1.0f / t;
  double lta = 0.0, lcd = 0.0;
  for (int b = 0; b < B; ++b) {
    float sa = 0.f, sc = 0.f;
    for (int i = threadIdx.x; i < per_sample; i += kTacdThreads) {
      const size_t k = (size_t)b * per_sample + i;
      const float at = a_t[k];
      const float uta = (at - a0_teacher[k]) * inv_t;
      const float vs = (at - f_student[k]) * inv_t;
      const float ucd = (at - f_ema[k]) * inv_t;
      if (u_ta) u_ta[k] = uta;
      if (v_student) v_student[k] = vs;
      if (u_cd) u_cd[k] = ucd;
      sa += (vs - uta) * (vs - uta);
      sc += (vs - ucd) * (vs - ucd);
    }
    red[0][threadIdx.x] = sa;
    red[1][threadIdx.x] = sc;
    __syncthreads();
    for (int w = kTacdThreads / 2; w > 0; w >>= 1) {
      if (threadIdx.x < w) {
        red[0][threadIdx.x] += red[0][threadIdx.x + w];
        red[1][threadIdx.x] += red[1][threadIdx.x + w];
      }
      __syncthreads();
    }
    if (threadIdx.x == 0) {
      lta += red[0][0];
      lcd += red[1][0];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const float l_ta = (float)(lta / B), l_cd = (float)(lcd / B);
    losses[0] = l_ta;
    losses[1] = l_cd;
    losses[2] = l_cd + lambda * l_ta;
  }
}

}  // namespace

cudaError_t launch_tacd_noise(const float* a_clean, const float* eps, float t, float* a_t, int n, cudaStream_t s) {
  const int grid = (n + 255) / 256 < 1 ? 1 : ((n + 255) / 256 > 148 ? 148 : (n + 255) / 256);
  return launch_k(tacd_noise_kernel, dim3(grid), dim3(256), 0, s, a_clean, eps, t, a_t, n);
}

cudaError_t launch_tacd_targets(const float* a_t, const float* a0_teacher, const float* f_student,
                                const float* f_ema, float t, float lambda, int B, int per_sample, float* u_ta,
                                float* v_student, float* u_cd, float* losses, cudaStream_t s) {
  return launch_k(tacd_targets_kernel, dim3(1), dim3(kTacdThreads), 0, s, a_t, a0_teacher, f_student, f_ema, t,
                  lambda, B, per_sample, u_ta, v_student, u_cd, losses);
}

}  // namespace wam
