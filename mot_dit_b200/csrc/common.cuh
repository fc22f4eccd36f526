// Device helpers shared by the sm_100a kernels of the MoT world-action-model
// library: bf16 packing, mbarriers with bounded waits, TMA tile loads, and the
// tcgen05 (5th-generation tensor core / tensor memory) primitives.
//
// Every wait in these kernels is bounded: a wait that does not complete within
// kWaitLimitNs of %globaltimer sets a bit in the caller-supplied status word and
// returns false, and the kernel then winds down (no trap, no endless spin).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace wam {

// Bits of the device status word (read back by the host as WAM_ERR_TIMEOUT).
enum : unsigned {
  kStatusTimeoutTmaFull = 1u << 0,   // MMA warp waited too long for a TMA stage
  kStatusTimeoutTmaEmpty = 1u << 1,  // producer waited too long for a free stage
  kStatusTimeoutAccum = 1u << 2,     // epilogue waited too long for the accumulator
  kStatusTimeoutDrain = 1u << 3,     // teardown waited too long for copies in flight
  kStatusTimeoutPeer = 1u << 4,      // waited too long for another CTA's partial tile
};

constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- bf16 ------
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ------------------------------------------------------------- mbarrier -----
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.  Returns false
// (and sets `bit` in *status) if it did not complete within kWaitLimitNs, or if
// another role of this CTA already failed (*abort set).  With abort == nullptr
// the wait ignores other roles' failures (used to drain copies in flight).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned* status,
                                          unsigned bit, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (abort && *abort) return false;
    if (globaltimer() - t0 > kWaitLimitNs) {
      atomicOr(status, bit);
      if (abort) *abort = 1;
      return false;
    }
  }
}

// ------------------------------------------------------------------ TMA -----
// 3-D tiled load (x = innermost element coordinate, y = row, z = matrix index)
// into shared memory, completing transaction bytes on `bar`.  No multicast.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// -------------------------------------------------------------- tcgen05 -----
__device__ __forceinline__ void tmem_alloc(uint32_t* slot_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(slot_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, both K-major, kind::f16 (bf16 in, f32 acc).
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once every tcgen05.mma issued so far by this thread completes.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets row
// (lane base + i), columns [col, col+32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor for a K-major bf16 tile stored as rows of
// 128 bytes (64 elements) with the 128-byte swizzle, 8-row groups 1024 B apart
// (the layout a TMA load with CU_TENSOR_MAP_SWIZZLE_128B produces).
__device__ __forceinline__ uint64_t smem_desc_k128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);  // start address
  d |= static_cast<uint64_t>(1) << 16;                // leading byte offset (unused, 16 B)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;        // stride byte offset: 8 rows x 128 B
  d |= static_cast<uint64_t>(1) << 46;                // descriptor version (sm_100)
  d |= static_cast<uint64_t>(2) << 61;                // layout: 128-byte swizzle
  return d;
}

// Instruction descriptor: bf16 x bf16 -> f32, both operands K-major, M x N tile.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int m, int n) {
  return (1u << 4)                                    // D format f32
         | (1u << 7)                                  // A format bf16
         | (1u << 10)                                 // B format bf16
         | (static_cast<uint32_t>(n >> 3) << 17)      // N / 8
         | (static_cast<uint32_t>(m >> 4) << 24);     // M / 16
}

// ------------------------------------------------- dependent launches -----
// Programmatic dependent launch: a kernel launched with the programmatic
// stream-serialization attribute may start before its predecessor on the
// stream finishes; it must call pdl_wait() before touching any global memory
// the predecessor writes or reads (both are no-ops without the attribute).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------ mma.sync -----
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* g, bool valid) {
  const int n = valid ? 16 : 0;  // zero-fill when invalid
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(saddr), "l"(g), "r"(n)
               : "memory");
}
// 16-byte async copy into shared memory, always valid source.
__device__ __forceinline__ void cp_async16_ca(uint32_t saddr, const void* g) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(g) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------ diagnostic kernel trace --
// Builds with -DWAM_KTRACE only: WAM_KTRACE_UNIT(name) in a .cu file gives it
// a record buffer and an extern "C" reader wam_debug_ktrace_<name>; the
// kernels there note their entry time (WAM_KT_BEGIN) and have thread 0 of
// every CTA append (kind, grid, block, SM, entry, exit) at its end (WAM_KT_END).
#ifdef WAM_KTRACE
struct KtRec {
  unsigned long long t0, t1;
  unsigned kind, grid_x, grid_y, block, smid, waited;  // waited: ns from entry to the dependent-launch wait's return
};
constexpr unsigned kKtMax = 1u << 18;
#define WAM_KTRACE_UNIT(name)                                                                           \
  __device__ KtRec g_kt_##name[kKtMax];                                                                 \
  __device__ unsigned g_kt_n_##name;                                                                    \
  __device__ __forceinline__ void kt_end_##name(unsigned long long t0, unsigned long long tw, unsigned kind) { \
    if (threadIdx.x != 0) return;                                                                        \
    const unsigned i = atomicAdd(&g_kt_n_##name, 1u);                                                    \
    if (i >= kKtMax) return;                                                                             \
    unsigned sm;                                                                                         \
    asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));                                                      \
    g_kt_##name[i] = KtRec{t0, globaltimer(), kind, gridDim.x, gridDim.y, blockIdx.x + 65536u * blockIdx.y, sm, \
                           (unsigned)(tw > t0 ? tw - t0 : 0)};                                           \
  }                                                                                                      \
  extern "C" int wam_debug_ktrace_##name(void* host, int cap) {                                          \
    unsigned n = 0;                                                                                      \
    if (cudaMemcpyFromSymbol(&n, g_kt_n_##name, 4) != cudaSuccess) return -1;                            \
    if (n > kKtMax) n = kKtMax;                                                                          \
    if ((int)n > cap) n = cap;                                                                           \
    if (n && cudaMemcpyFromSymbol(host, g_kt_##name, n * sizeof(KtRec)) != cudaSuccess) return -1;       \
    const unsigned z = 0;                                                                                \
    cudaMemcpyToSymbol(g_kt_n_##name, &z, 4);                                                            \
    return (int)n;                                                                                       \
  }
#define WAM_KT_BEGIN                            \
  const unsigned long long kt_t0 = globaltimer(); \
  unsigned long long kt_tw = 0
#define WAM_KT_WAITED() (kt_tw = globaltimer())
#define WAM_KT_END(name, kind) kt_end_##name(kt_t0, kt_tw, (kind))
#else
#define WAM_KTRACE_UNIT(name)
#define WAM_KT_BEGIN
#define WAM_KT_WAITED()
#define WAM_KT_END(name, kind)
#endif

// ------------------------------------------------- norm + modulation -------
// One row, one warp: h = rms(x) * (gain ? gain[n] : 1 + scale[n]) + (shift ?
// shift[n] : 0), rms(x) = x / sqrt(mean(x^2) + 1e-6).  A lane holds up to
// kRowNormV float4 of the row in registers so every load of the row is in
// flight at once (d a multiple of 4, d <= 32 * 4 * kRowNormV).  Every place
// that normalises a row calls this, so all of them round alike.
constexpr int kRowNormV = 12;

// The row's values (every load issued before any is used).
__device__ __forceinline__ void norm_row_load(const float* __restrict__ x, int d, int lane, float4 (&v)[kRowNormV]) {
  const float4* xr = reinterpret_cast<const float4*>(x);
  const int n4 = d >> 2;
#pragma unroll
  for (int k = 0; k < kRowNormV; ++k) {
    const int i = lane + 32 * k;
    v[k] = i < n4 ? xr[i] : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}
// 1 / rms of the row (lane partial sums in k order, then a xor-shuffle tree).
__device__ __forceinline__ float norm_row_rscale(const float4 (&v)[kRowNormV], int d) {
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < kRowNormV; ++k) ss += v[k].x * v[k].x + v[k].y * v[k].y + v[k].z * v[k].z + v[k].w * v[k].w;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  return 1.0f / sqrtf(ss / (float)d + 1e-6f);
}
// h = v * r * mul + add, with mul / add the modulation's float4 i (mul
// already 1 + scale, or the gain).
template <bool BF16, typename MulAdd>
__device__ __forceinline__ void norm_row_store(const float4 (&v)[kRowNormV], float r, int d, int lane, void* __restrict__ h,
                                               MulAdd mul_add) {
  const int n4 = d >> 2;
#pragma unroll
  for (int k = 0; k < kRowNormV; ++k) {
    const int i = lane + 32 * k;
    if (i >= n4) break;
    float4 mul4, add4;
    mul_add(i, mul4, add4);
    float y[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
    y[0] = y[0] * r * mul4.x + add4.x;
    y[1] = y[1] * r * mul4.y + add4.y;
    y[2] = y[2] * r * mul4.z + add4.z;
    y[3] = y[3] * r * mul4.w + add4.w;
    if (BF16) {
      uint2 p;
      p.x = pack_bf16(y[0], y[1]);
      p.y = pack_bf16(y[2], y[3]);
      reinterpret_cast<uint2*>(h)[i] = p;
    } else {
      reinterpret_cast<float4*>(h)[i] = make_float4(y[0], y[1], y[2], y[3]);
    }
  }
}
// The modulation's float4 i: (gain or 1 + scale, shift or 0).
__device__ __forceinline__ void norm_mod_vec(const float* __restrict__ scale, const float* __restrict__ shift,
                                             const float* __restrict__ gain, int i, float4& mul4, float4& add4) {
  if (gain) {
    mul4 = __ldg(reinterpret_cast<const float4*>(gain) + i);
  } else {
    mul4 = __ldg(reinterpret_cast<const float4*>(scale) + i);
    mul4.x += 1.f;
    mul4.y += 1.f;
    mul4.z += 1.f;
    mul4.w += 1.f;
  }
  add4 = shift ? __ldg(reinterpret_cast<const float4*>(shift) + i) : make_float4(0.f, 0.f, 0.f, 0.f);
}

template <bool BF16>
__device__ __forceinline__ void norm_mod_row(const float* __restrict__ x, void* __restrict__ h, int d,
                                             const float* __restrict__ scale, const float* __restrict__ shift,
                                             const float* __restrict__ gain, int lane) {
  float4 v[kRowNormV];
  norm_row_load(x, d, lane, v);
  const float r = norm_row_rscale(v, d);
  norm_row_store<BF16>(v, r, d, lane, h, [&](int i, float4& m, float4& a) { norm_mod_vec(scale, shift, gain, i, m, a); });
}

// GELU, tanh form: 0.5 x (1 + tanh(z)), z = sqrt(2/pi) (x + 0.044715 x^3),
// evaluated through the identity 0.5 (1 + tanh(z)) = 1 / (1 + exp(-2 z)).
__device__ __forceinline__ float gelu_tanh(float x) {
  const float k2 = 1.5957691216057308f;  // 2 sqrt(2/pi)
  const float z2 = k2 * (x + 0.044715f * x * x * x);
  return __fdividef(x, 1.0f + __expf(-z2));
}

}  // namespace wam
