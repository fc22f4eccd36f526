// Small kernels of the MoT world-action-model path: the RMSNorm / AdaLN
// modulation prologue, the timestep conditioning (three GEMVs), chunk input
// and output movers, the joint variant's noising, the seeded parameter
// generator and the RoPE table.  Also the TMA tensor-map factory.
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstdlib>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace wam {
namespace {

constexpr int kNormWarps = 16;      // rows per CTA (config-2 chunk 4.09 -> 4.02 ms against 8)
constexpr int kNormWarpsSmall = 4;  // rows per CTA up to kNormSmallRows rows, so more SMs share the loads
constexpr int kNormSmallRows = 256;

}  // namespace
WAM_KTRACE_UNIT(misc)
namespace {

// ------------------------------------------------- norm + modulation -------
// One warp per row (norm_mod_row, shared with the fused-norm GEMM prologue),
// WARPS rows per CTA.
template <bool BF16, int WARPS>
__global__ void __launch_bounds__(32 * WARPS)
    norm_mod_kernel(const float* __restrict__ x, void* __restrict__ h, int M, int d, const float* __restrict__ scale,
                    const float* __restrict__ shift, const float* __restrict__ gain, int ldh) {
  // the modulation vectors, shared by every row of the CTA
  __shared__ float4 s_mul[kRowNormMax / 4];
  __shared__ float4 s_add[kRowNormMax / 4];
  WAM_KT_BEGIN;
  pdl_trigger();
  pdl_wait();
  WAM_KT_WAITED();
  const int row = blockIdx.x * WARPS + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const bool has_row = row < M;
  // one round trip: the row's loads go out first, then the CTA stages the
  // modulation vectors while they are in flight
  float4 v[kRowNormV];
  norm_row_load(x + (size_t)(has_row ? row : 0) * d, d, lane, v);
  for (int i = threadIdx.x; i < (d >> 2); i += blockDim.x) norm_mod_vec(scale, shift, gain, i, s_mul[i], s_add[i]);
  __syncthreads();
  if (!has_row) return;
  const float r = norm_row_rscale(v, d);
  norm_row_store<BF16>(v, r, d, lane,
                       BF16 ? (void*)(reinterpret_cast<__nv_bfloat16*>(h) + (size_t)row * ldh)
                            : (void*)(reinterpret_cast<float*>(h) + (size_t)row * ldh),
                       [&](int i, float4& m, float4& a) {
                         m = s_mul[i];
                         a = s_add[i];
                       });
  WAM_KT_END(misc, 2u);
}

// ------------------------------------------------ timestep conditioning ----
// y[n] = sum_k W[n, k] f(x[k]) + b[n] with f = identity / SiLU, or with x the
// 256 sinusoidal features of the device scalar t (mode 2).  With `mod`, the
// result is written as mod[i, n] = y[n] + T_i[n] for every block i.
constexpr int kGemvWarps = 8;

__device__ __forceinline__ float silu(float v) { return v / (1.0f + expf(-v)); }

template <bool BF16>
__global__ void __launch_bounds__(32 * kGemvWarps)
    gemv_kernel(const void* __restrict__ W, const float* __restrict__ x, const float* __restrict__ t, int mode,
                const float* __restrict__ bias, float* __restrict__ y, int N, int K, const float* __restrict__ T0,
                size_t T_stride, int n_blocks, float* __restrict__ mod, int* set_flag) {
  extern __shared__ float xs[];
  pdl_trigger();
  pdl_wait();
  // every kernel before this one on the stream is complete and its writes
  // visible: say so to later kernels that read before their own wait
  if (set_flag && blockIdx.x == 0 && threadIdx.x == 0)
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(set_flag), "r"(1) : "memory");
  if (mode == 2) {
    const double tt = (double)t[0];
    for (int k = threadIdx.x; k < 128; k += blockDim.x) {
      const double w = pow(10000.0, -(double)k / 128.0);
      const double arg = 1000.0 * tt * w;
      xs[k] = (float)cos(arg);
      xs[k + 128] = (float)sin(arg);
    }
  } else {
    for (int k = threadIdx.x; k < K; k += blockDim.x) xs[k] = mode == 1 ? silu(x[k]) : x[k];
  }
  __syncthreads();
  const int n = blockIdx.x * kGemvWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (n >= N) return;
  float acc = 0.f;
  if (BF16) {
    const uint4* wr = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(W) + (size_t)n * K);
    for (int c = lane; c < K / 8; c += 32) {
      const uint4 w4 = __ldg(wr + c);
      const __nv_bfloat162* wp = reinterpret_cast<const __nv_bfloat162*>(&w4);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 wf = __bfloat1622float2(wp[j]);
        acc += wf.x * xs[8 * c + 2 * j] + wf.y * xs[8 * c + 2 * j + 1];
      }
    }
  } else {
    const float4* wr = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(W) + (size_t)n * K);
    for (int c = lane; c < K / 4; c += 32) {
      const float4 w4 = __ldg(wr + c);
      acc += w4.x * xs[4 * c] + w4.y * xs[4 * c + 1] + w4.z * xs[4 * c + 2] + w4.w * xs[4 * c + 3];
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) {
    const float v = acc + bias[n];
    if (mod) {
      for (int i = 0; i < n_blocks; ++i) mod[(size_t)i * N + n] = v + T0[i * T_stride + n];
    } else {
      y[n] = v;
    }
  }
}

// --------------------------------------------------------- io movers -------
__global__ void set_video_io_kernel(VideoIo* dst, VideoIo v) {
  if (v.shift > 0.f) {
    const double u = v.u, s = v.shift;
    v.t = (float)(s * u / (1.0 + (s - 1.0) * u));
  }
  *dst = v;
}

__global__ void set_action_io_kernel(ActionIo* dst, ActionIo v) {
  if (v.shift > 0.f) {
    const double u = v.u, s = v.shift;
    v.sched[0] = (float)(s * u / (1.0 + (s - 1.0) * u));
    v.sched[1] = 0.f;
    v.steps = 1;
  }
  *dst = v;
}

__global__ void init_video_kernel(const VideoIo* __restrict__ io, float* __restrict__ x, int B, int Lc, int Lvid,
                                  int d) {
  pdl_trigger();
  pdl_wait();
  const size_t n = (size_t)B * (Lc + Lvid) * d;
  const float* video = io->video;
  const float* cond = io->cond;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const size_t row = i / d, c = i % d;
    const int b = (int)(row / (Lc + Lvid)), l = (int)(row % (Lc + Lvid));
    x[i] = l < Lc ? cond[((size_t)b * Lc + l) * d + c] : video[((size_t)b * Lvid + (l - Lc)) * d + c];
  }
}

__device__ __forceinline__ void write_in(void* a_in, bool bf16, size_t idx, float v) {
  if (bf16)
    reinterpret_cast<__nv_bfloat16*>(a_in)[idx] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float*>(a_in)[idx] = v;
}

__global__ void init_action_kernel(const ActionIo* __restrict__ io, float* __restrict__ a_state, void* a_in,
                                   int bf16, int M, int P, int ld_in) {
  pdl_trigger();
  pdl_wait();
  const float* src = io->a_in;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < M * P; i += gridDim.x * blockDim.x) {
    const float v = src[i];
    a_state[i] = v;
    if (a_in) write_in(a_in, bf16, (size_t)(i / P) * ld_in + i % P, v);
  }
}

__global__ void noise_action_kernel(const ActionIo* __restrict__ io, float* __restrict__ a_state, void* a_in,
                                    int bf16, int M, int P, int ld_in) {
  pdl_trigger();
  pdl_wait();
  const float sigma = io->sched[0];
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < M * P; i += gridDim.x * blockDim.x) {
    const float v = (1.0f - sigma) * io->a_clean[i] + sigma * io->a_in[i];
    a_state[i] = v;
    if (a_in) write_in(a_in, bf16, (size_t)(i / P) * ld_in + i % P, v);
  }
}

__global__ void noise_video_kernel(const VideoIo* __restrict__ io, float* __restrict__ xs, void* x_act, int bf16,
                                   int n_rows, int P, int ld_act) {
  pdl_trigger();
  pdl_wait();
  const float sigma = io->t;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_rows * P; i += gridDim.x * blockDim.x) {
    const float v = (1.0f - sigma) * io->video[i] + sigma * io->eps[i];
    xs[i] = v;
    write_in(x_act, bf16, (size_t)(i / P) * ld_act + i % P, v);
  }
}

__global__ void copy_out_kernel(const ActionIo* __restrict__ io, const float* __restrict__ a, int n) {
  pdl_trigger();
  pdl_wait();
  float* out = io->a_out;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) out[i] = a[i];
}

// ------------------------------------------------------ pixel front-end -----
// Patchify / unpatchify of channel-first frames [B, F, C, H, W] <-> patch
// tokens [B, F (H/p)(W/p), C p p] (token = frame-major raster order of the
// patches, feature = (channel, row, column) within the patch).  One thread
// per patch-token element; the patch side is written (patchify) or read
// (unpatchify) contiguously.
__global__ void patchify_kernel(const float* __restrict__ src, float* __restrict__ dst, int F, int C, int H, int W,
                                int p, size_t n, int inverse) {
  pdl_trigger();
  pdl_wait();
  const int Hp = H / p, Wp = W / p, cpp = C * p * p;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const size_t tok = i / cpp;
    const int feat = (int)(i - tok * cpp);
    const int per_sample = F * Hp * Wp;
    const size_t b = tok / per_sample;
    const int t = (int)(tok - b * per_sample);
    const int f = t / (Hp * Wp), py = (t / Wp) % Hp, px = t % Wp;
    const int c = feat / (p * p), iy = (feat / p) % p, ix = feat % p;
    const size_t pix = ((((b * F + f) * C + c) * (size_t)H + (py * p + iy)) * W) + px * p + ix;
    if (inverse)
      dst[pix] = src[i];
    else
      dst[i] = src[pix];
  }
}

// -------------------------------------------------- seeded parameters ------
__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__global__ void gen_param_kernel(uint64_t seed, uint64_t pid, size_t count, double stdv, int ones, int round_bf16,
                                 void* out, int out_bf16, int cols, int ld) {
  const uint64_t key = seed ^ (pid * 0x9E3779B97F4A7C15ull);
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < count; e += (size_t)gridDim.x * blockDim.x) {
    float f;
    if (ones) {
      f = 1.0f;
    } else {
      const uint64_t c0 = key + 2ull * e;
      const double u0 = (double)((splitmix64(c0) >> 11) + 1) * 0x1p-53;
      const double u1 = (double)((splitmix64(c0 + 1) >> 11) + 1) * 0x1p-53;
      const double z = sqrt(-2.0 * log(u0)) * cos(2.0 * 3.141592653589793 * u1);
      f = __double2float_rn(stdv * z);
    }
    if (round_bf16) f = __bfloat162float(__float2bfloat16_rn(f));
    const size_t idx = (e / cols) * ld + e % cols;
    if (out_bf16)
      reinterpret_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(f);
    else
      reinterpret_cast<float*>(out)[idx] = f;
  }
}

__global__ void rope_table_kernel(float* cos_t, float* sin_t, int L, int Dh) {
  const int half = Dh / 2;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < L * half; i += gridDim.x * blockDim.x) {
    const int pos = i / half, j = i % half;
    const double theta = (double)pos * pow(10000.0, -2.0 * j / Dh);
    cos_t[i] = (float)cos(theta);
    sin_t[i] = (float)sin(theta);
  }
}

__global__ void to_f32_kernel(const void* src, int bf16, float* dst, size_t n, int cols, int ld) {
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
    const size_t idx = (e / cols) * ld + e % cols;
    dst[e] = bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(src)[idx])
                  : reinterpret_cast<const float*>(src)[idx];
  }
}

int grid_for(size_t n, int threads) {
  size_t b = (n + threads - 1) / threads;
  if (b > 148 * 16) b = 148 * 16;
  return b < 1 ? 1 : (int)b;
}

}  // namespace

cudaError_t launch_norm_mod(const float* x, void* h, bool h_bf16, int M, int d, const float* scale,
                            const float* shift, const float* gain, cudaStream_t s, int ldh) {
  if (ldh == 0) ldh = d;
  if (ldh < d || ldh % 4) return cudaErrorInvalidValue;
  if (d % 4 != 0 || d > 32 * 4 * kRowNormV) return cudaErrorInvalidValue;
  if (M <= kNormSmallRows) {
    const dim3 grid((M + kNormWarpsSmall - 1) / kNormWarpsSmall), block(32 * kNormWarpsSmall);
    if (h_bf16) return launch_k(norm_mod_kernel<true, kNormWarpsSmall>, grid, block, 0, s, x, h, M, d, scale, shift, gain, ldh);
    return launch_k(norm_mod_kernel<false, kNormWarpsSmall>, grid, block, 0, s, x, h, M, d, scale, shift, gain, ldh);
  }
  const dim3 grid((M + kNormWarps - 1) / kNormWarps), block(32 * kNormWarps);
  if (h_bf16) return launch_k(norm_mod_kernel<true, kNormWarps>, grid, block, 0, s, x, h, M, d, scale, shift, gain, ldh);
  return launch_k(norm_mod_kernel<false, kNormWarps>, grid, block, 0, s, x, h, M, d, scale, shift, gain, ldh);
}

cudaError_t launch_temb(const TembArgs& a, cudaStream_t s) {
  const int d = a.d;
  if (d % 8 != 0) return cudaErrorInvalidValue;
  float* c1 = a.scratch;
  float* c = a.scratch + d;
  auto gemv = [&](const void* W, const float* x, int mode, const float* b, float* y, int N, int K, bool mod,
                  int* flag = nullptr) {
    dim3 grid((N + kGemvWarps - 1) / kGemvWarps);
    const size_t sm = (size_t)(mode == 2 ? 256 : K) * sizeof(float);
    float* modp = mod ? a.mod : nullptr;
    if (a.bf16)
      return launch_k(gemv_kernel<true>, grid, dim3(32 * kGemvWarps), sm, s, W, x, a.t, mode, b, y, N, K, a.T0,
                      a.T_stride, a.n_blocks, modp, flag);
    return launch_k(gemv_kernel<false>, grid, dim3(32 * kGemvWarps), sm, s, W, x, a.t, mode, b, y, N, K, a.T0,
                    a.T_stride, a.n_blocks, modp, flag);
  };
  cudaError_t e;
  if ((e = gemv(a.w1, nullptr, 2, a.b1, c1, d, 256, false, a.set_flag)) != cudaSuccess) return e;
  if ((e = gemv(a.w2, c1, 1, a.b2, c, d, d, false)) != cudaSuccess) return e;
  return gemv(a.wm, c, 1, a.bm, nullptr, 6 * d, d, true);
}

cudaError_t launch_init_video(const VideoIo* io, float* x, int B, int Lc, int Lvid, int d, cudaStream_t s) {
  const size_t n = (size_t)B * (Lc + Lvid) * d;
  return launch_k(init_video_kernel, dim3(grid_for(n, 256)), dim3(256), 0, s, io, x, B, Lc, Lvid, d);
}

cudaError_t launch_init_action(const ActionIo* io, float* a_state, void* a_in, bool a_in_bf16, int M, int P,
                               int ld_in, cudaStream_t s) {
  return launch_k(init_action_kernel, dim3(grid_for((size_t)M * P, 256)), dim3(256), 0, s, io, a_state, a_in,
                  (int)a_in_bf16, M, P, ld_in);
}

cudaError_t launch_noise_action(const ActionIo* io, float* a_state, void* a_in, bool a_in_bf16, int M, int P,
                                int ld_in, cudaStream_t s) {
  return launch_k(noise_action_kernel, dim3(grid_for((size_t)M * P, 256)), dim3(256), 0, s, io, a_state, a_in,
                  (int)a_in_bf16, M, P, ld_in);
}

cudaError_t launch_noise_video(const VideoIo* io, float* x_sigma, void* x_act, bool act_bf16, int n_rows, int P,
                               int ld_act, cudaStream_t s) {
  return launch_k(noise_video_kernel, dim3(grid_for((size_t)n_rows * P, 256)), dim3(256), 0, s, io, x_sigma, x_act,
                  (int)act_bf16, n_rows, P, ld_act);
}

cudaError_t launch_patchify(const float* src, float* dst, int B, int F, int C, int H, int W, int p, bool inverse,
                            cudaStream_t s) {
  const size_t n = (size_t)B * F * C * H * W;
  return launch_k(patchify_kernel, dim3(grid_for(n, 256)), dim3(256), 0, s, src, dst, F, C, H, W, p, n,
                  inverse ? 1 : 0);
}

cudaError_t launch_copy_out(const ActionIo* io, const float* a_state, int n, cudaStream_t s) {
  return launch_k(copy_out_kernel, dim3(grid_for(n, 256)), dim3(256), 0, s, io, a_state, n);
}

cudaError_t launch_set_video_io(VideoIo* dst, const VideoIo& v, cudaStream_t s) {
  set_video_io_kernel<<<1, 1, 0, s>>>(dst, v);
  return cudaGetLastError();
}

cudaError_t launch_set_action_io(ActionIo* dst, const ActionIo& v, cudaStream_t s) {
  set_action_io_kernel<<<1, 1, 0, s>>>(dst, v);
  return cudaGetLastError();
}

cudaError_t launch_gen_param(uint64_t seed, uint64_t pid, size_t count, double stdv, bool ones, bool round_bf16,
                             void* out, bool out_bf16, int cols, int ld, cudaStream_t s) {
  gen_param_kernel<<<grid_for(count, 256), 256, 0, s>>>(seed, pid, count, stdv, ones, round_bf16, out, out_bf16,
                                                         cols, ld);
  return cudaGetLastError();
}

cudaError_t launch_rope_table(float* cos_t, float* sin_t, int L, int Dh, cudaStream_t s) {
  rope_table_kernel<<<grid_for((size_t)L * Dh / 2, 256), 256, 0, s>>>(cos_t, sin_t, L, Dh);
  return cudaGetLastError();
}

cudaError_t launch_to_f32(const void* src, bool src_bf16, float* dst, size_t n, int cols, int ld, cudaStream_t s) {
  to_f32_kernel<<<grid_for(n, 256), 256, 0, s>>>(src, src_bf16, dst, n, cols, ld);
  return cudaGetLastError();
}

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = getenv("WAM_PDL");
    return !(v && v[0] == '0');
  }();
  return on;
}

// ------------------------------------------------------- tensor maps -------
namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
}  // namespace

static bool encoder_ready();

bool make_tmap_sw128(CUtensorMap* map, const void* base, int elem_bytes, int inner, int rows, int nmat,
                     size_t mat_stride_bytes, int box_inner, int box_rows) {
  if (!encoder_ready()) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || ((size_t)inner * elem_bytes) % 16 || mat_stride_bytes % 16 ||
      box_inner * elem_bytes != 128)
    return false;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)nmat};
  cuuint64_t strides[2] = {(cuuint64_t)inner * elem_bytes,
                           (cuuint64_t)(nmat > 1 ? mat_stride_bytes : (size_t)inner * elem_bytes * rows)};
  cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, elem_bytes == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                        const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static bool encoder_ready() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

bool make_tmap_3d(CUtensorMap* map, const void* base, int K, int rows, int nmat, size_t mat_stride_bytes,
                  int box_rows) {
  if (!encoder_ready()) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || ((size_t)K * 2) % 16 || mat_stride_bytes % 16) return false;
  cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)rows, (cuuint64_t)nmat};
  cuuint64_t strides[2] = {(cuuint64_t)K * 2, (cuuint64_t)(nmat > 1 ? mat_stride_bytes : (size_t)K * 2 * rows)};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace wam
