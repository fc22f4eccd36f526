// Video-query attention on the 5th-generation tensor cores (tcgen05).
//
// softmax(Q K^T / sqrt(64)) V for one (sample, head) and 128 queries per CTA,
// over keys [0, Lk) of the per-block cache (the video expert's own keys;
// RealtimeWAM summary page, 前置知识 "Mixture-of-Transformers": video queries
// see video keys only).
//
// Two independent flash-attention streams share one CTA: softmax warpgroup g
// (g = 0, 1) owns the key tiles j = g, g + 2, g + 4, ... (64 keys each), with
// its own S buffer, P buffer, O accumulator, row maximum and row sum; the two
// are merged at the end (log-sum-exp weights, as for split keys).  For tile j
// of stream g:
//   S_j  = Q K_j^T      tcgen05.mma M=128 N=64 K=64, fp32 into TMEM S_g
//   P_j  = exp2(S_j log2e / 8 - m_g)   thread = query row (64 keys), bf16
//          pairs written back over the first 32 columns of S_g (tcgen05.st)
//   O_g += P_j V_j      tcgen05.mma M=128 N=64 K=64 accumulating in TMEM, P
//          as the A operand straight from TMEM, V as the MN-major B operand
//          from shared memory (the cache rows are [key][64 channels])
// m_g is raised (and O_g and the row sum rescaled in place) only when a tile's
// maximum exceeds it by more than 2^8: exact softmax arithmetic with a stale
// maximum, P <= 256, and in most tiles no TMEM round trip of O.  The MMA warp
// issues S_{j+2} right after PV_j, so while one warpgroup exponentiates tile
// j the tensor core already holds the other's tile j+1 and its own tile j+2;
// K/V tiles are 4-stage buffered by TMA.
//
// Warp roles (320 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA
// issuer, warps 2..9 softmax: warp w reads TMEM lanes 32*(w%4)..+31 (its 32
// query rows) of its warpgroup (w-2)/4's S and O columns.
// Every wait is bounded (see common.cuh).
#include "common.cuh"
#include "kernels.h"

namespace wam {
namespace {

constexpr int kQ = 128;       // queries per CTA
constexpr int kKT = 64;       // keys per tile
constexpr int kDh = 64;
constexpr int kStagesKV = 4;
constexpr int kQBytes = kQ * kDh * 2;      // 16 KB
constexpr int kKVBytes = kKT * kDh * 2;    // 8 KB (one K or V tile)
constexpr int kXchBytes = 3 * kQ * 4;      // stream 1's (m, l, ok) per row for the final merge
constexpr int kThreads = 320;              // producer, MMA, two softmax warpgroups
constexpr int kTmemCols = 256;             // S_0 [0,64), S_1 [64,128), O_0 [128,192), O_1 [192,256)
constexpr float kRescale = 8.0f;           // log2 headroom of the stale row maximum
constexpr int kBarBytes = 128;
// No alignment slack: two CTAs per SM need every byte (2 x (112 KB + 1 KB reserved) <= 228 KB).
constexpr int kSmem = kQBytes + kStagesKV * 2 * kKVBytes + kXchBytes + kBarBytes;

// Shared-memory descriptor of an MN-major bf16 operand stored as rows of 128
// bytes (64 elements along N) with the 128-byte swizzle, consecutive K rows
// 128 B apart, 8-row groups 1024 B apart (a TMA SWIZZLE_128B tile of [K][64]).
__device__ __forceinline__ uint64_t smem_desc_mn128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);  // start address
  d |= static_cast<uint64_t>(1) << 16;                // leading byte offset (one 64-wide atom: unused)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;        // stride byte offset: 8 K-rows x 128 B
  d |= static_cast<uint64_t>(1) << 46;                // descriptor version (sm_100)
  d |= static_cast<uint64_t>(2) << 61;                // layout: 128-byte swizzle
  return d;
}

__device__ __forceinline__ void mbar_arrive_cta(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns from registers, one wait.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]: the A operand (M = 128 rows on the TMEM
// lanes, K-major, two 16-bit elements per 32-bit column) read from tensor memory.
__device__ __forceinline__ void tc_mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 64 consecutive 32-bit columns, one wait.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
  uint32_t r[64];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 lanes x 64 columns back into TMEM, one wait.
__device__ __forceinline__ void tmem_st64(uint32_t taddr, const float (&v)[64]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,"
      "%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,"
      "%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]), "f"(v[9]),
      "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]), "f"(v[16]), "f"(v[17]), "f"(v[18]),
      "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]), "f"(v[24]), "f"(v[25]), "f"(v[26]), "f"(v[27]),
      "f"(v[28]), "f"(v[29]), "f"(v[30]), "f"(v[31]), "f"(v[32]), "f"(v[33]), "f"(v[34]), "f"(v[35]), "f"(v[36]),
      "f"(v[37]), "f"(v[38]), "f"(v[39]), "f"(v[40]), "f"(v[41]), "f"(v[42]), "f"(v[43]), "f"(v[44]), "f"(v[45]),
      "f"(v[46]), "f"(v[47]), "f"(v[48]), "f"(v[49]), "f"(v[50]), "f"(v[51]), "f"(v[52]), "f"(v[53]), "f"(v[54]),
      "f"(v[55]), "f"(v[56]), "f"(v[57]), "f"(v[58]), "f"(v[59]), "f"(v[60]), "f"(v[61]), "f"(v[62]), "f"(v[63])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// max(a, b, c) in one instruction.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x on the special-function unit (the hardware approximation, flushing
// denormal results to zero; its relative error is far below bf16 rounding).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace
WAM_KTRACE_UNIT(attn)
namespace {

struct AttnTcK {
  int H, Lq, Lk, B;
  int zq0, zk0, zv0;  // z (matrix) index of (b=0, h=0) in the Q / K / V maps
  __nv_bfloat16* out;  // [B*Lq, H*64]
  unsigned* status;
};

__global__ void __launch_bounds__(kThreads, 2)
    attn_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v, const AttnTcK a) {
  WAM_KT_BEGIN;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // The 128-byte swizzle pattern is a function of the address bits: every tile
  // must start on a 1024-byte boundary.
  if (smem_u32(smem_raw) & 1023) {
    if (threadIdx.x == 0) atomicOr(a.status, kStatusTimeoutDrain);
    return;
  }
  uint8_t* sQ = smem_raw;
  uint8_t* sK = sQ + kQBytes;                  // [stage] K tiles
  uint8_t* sV = sK + kStagesKV * kKVBytes;     // [stage] V tiles
  float* xch = reinterpret_cast<float*>(sV + kStagesKV * kKVBytes);  // [128] m_1, [128] l_1, [128] ok_1
  uint64_t* bar = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(xch) + kXchBytes);
  uint64_t* q_full = bar + 0;
  uint64_t* kv_full = bar + 1;   // [4]
  uint64_t* kv_empty = bar + 5;  // [4]
  uint64_t* s_full = bar + 9;    // [2] S_g written (MMA -> softmax g)
  uint64_t* p_full = bar + 11;   // [2] P_g written, S_g read (softmax g -> MMA)
  uint64_t* pv_full = bar + 13;  // [2] PV into O_g complete (MMA -> softmax g)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 15);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * kQ, h = blockIdx.y, b = blockIdx.z;
  const int bh = b * a.H + h;
  const int ntiles = (a.Lk + kKT - 1) / kKT;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStagesKV; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(&s_full[g], 1);
      mbar_init(&p_full[g], 128);
      mbar_init(&pv_full[g], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&map_q);
    prefetch_tensormap(&map_k);
    prefetch_tensormap(&map_v);
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
    if (lane == 0) {
      pdl_wait();
      WAM_KT_WAITED();
      mbar_arrive_expect_tx(q_full, kQBytes);
      tma_load_3d(sQ, &map_q, q_full, 0, q0, a.zq0 + bh);
      int issued = 0;
      for (int j = 0; j < ntiles; ++j) {
        const int s = j % kStagesKV;
        if (j >= kStagesKV &&
            !mbar_wait(&kv_empty[s], ((j / kStagesKV) - 1) & 1, a.status, kStatusTimeoutTmaEmpty, abort_flag))
          break;
        mbar_arrive_expect_tx(&kv_full[s], 2 * kKVBytes);
        tma_load_3d(sK + s * kKVBytes, &map_k, &kv_full[s], 0, j * kKT, a.zk0 + bh);
        tma_load_3d(sV + s * kKVBytes, &map_v, &kv_full[s], 0, j * kKT, a.zv0 + bh);
        issued = j + 1;
      }
      mbar_wait(q_full, 0, a.status, kStatusTimeoutDrain, nullptr);
      for (int j = max(0, issued - kStagesKV); j < issued; ++j)
        mbar_wait(&kv_full[j % kStagesKV], (j / kStagesKV) & 1, a.status, kStatusTimeoutDrain, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kQ, kKT);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kQ, kDh) | (1u << 16);  // B (V) is MN-major
      const uint32_t aq = smem_u32(sQ);
      // S_j into S_{j & 1} (TMEM columns 64 (j & 1) ..)
      auto issue_s = [&](int j) {
        const int s = j % kStagesKV;
        if (!mbar_wait(&kv_full[s], (j / kStagesKV) & 1, a.status, kStatusTimeoutTmaFull, abort_flag)) return false;
        tc_fence_after();
        const uint32_t ak = smem_u32(sK + s * kKVBytes);
#pragma unroll
        for (int kk = 0; kk < kDh / 16; ++kk)
          tc_mma_bf16(tmem + (j & 1) * kKT, smem_desc_k128(aq + kk * 32), smem_desc_k128(ak + kk * 32), idesc_s,
                      kk > 0 ? 1u : 0u);
        tc_commit(&s_full[j & 1]);
        return true;
      };
      bool ok = mbar_wait(q_full, 0, a.status, kStatusTimeoutTmaFull, abort_flag);
      ok = ok && issue_s(0);
      if (ntiles > 1) ok = ok && issue_s(1);
      for (int j = 0; j < ntiles && ok; ++j) {
        const int g = j & 1, t = j >> 1;  // stream, its tile count
        // P_j written (and S_j read) by softmax warpgroup g
        if (!mbar_wait(&p_full[g], t & 1, a.status, kStatusTimeoutAccum, abort_flag)) break;
        tc_fence_after();
        const int s = j % kStagesKV;
        const uint32_t av = smem_u32(sV + s * kKVBytes);
        // P_j sits in the first 32 columns of S_g (16 keys = 8 columns a step);
        // S_{j+2}, issued after this, overwrites it only once these have read it
#pragma unroll
        for (int kk = 0; kk < kKT / 16; ++kk)
          tc_mma_bf16_ts(tmem + 128 + g * kDh, tmem + g * kKT + kk * 8, smem_desc_mn128(av + kk * 16 * 128),
                         idesc_pv, (t > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&pv_full[g]);
        tc_commit(&kv_empty[s]);  // K_j and V_j are read
        if (j + 2 < ntiles && !issue_s(j + 2)) break;
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ softmax warps
    pdl_wait();
    const int quad = warp & 3;
    const int g = (warp - 2) >> 2;   // stream: key tiles g, g + 2, ...
    const int r = quad * 32 + lane;  // query row within the tile
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t t_s = t_lane + g * kKT, t_o = t_lane + 128 + g * kDh;
    const float sl2e = 1.4426950408889634f * 0.125f;  // log2(e) / sqrt(64)
    float mref = -INFINITY, l = 0.f;  // reference maximum (scaled log2 units) and row sum of the stream
    bool ok = true;
    int t = 0;
    for (int j = g; j < ntiles; j += 2, ++t) {
      if (!mbar_wait(&s_full[g], t & 1, a.status, kStatusTimeoutAccum, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int nvalid = min(kKT, a.Lk - j * kKT);  // keys of this tile inside [0, Lk) (>= 1)
      float mx = -INFINITY;
      {
        float v[64];
        tmem_ld64(t_s, v);
        if (nvalid == kKT) {
#pragma unroll
          for (int i = 0; i < 64; i += 2) mx = fmax3(mx, v[i], v[i + 1]);
        } else {
#pragma unroll
          for (int i = 0; i < 64; ++i)
            if (i < nvalid) mx = fmaxf(mx, v[i]);
        }
      }
      const float mxs = mx * sl2e;
      if (t == 0) {
        mref = mxs;  // O_g is written from scratch by the stream's first PV
      } else {
        // PV of the stream's previous tile still reads P_g: wait for it before
        // P_j overwrites it (and before O_g may be rescaled)
        const bool got = mbar_wait(&pv_full[g], (t - 1) & 1, a.status, kStatusTimeoutAccum, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {  // leave together: the TMEM accesses below are warp-wide
          ok = false;
          break;
        }
        tc_fence_after();
        const bool need = mxs > mref + kRescale;
        if (__any_sync(0xffffffffu, need)) {  // tcgen05.ld / st are warp-wide
          const float alpha = need ? ex2(mref - mxs) : 1.f;
          if (need) mref = mxs;
          float o[64];
          tmem_ld64(t_o, o);
#pragma unroll
          for (int i = 0; i < kDh; ++i) o[i] *= alpha;
          tmem_st64(t_o, o);
          l *= alpha;
        }
      }
      float rs = 0.f;
      float v[64];
      tmem_ld64(t_s, v);
      if (nvalid == kKT) {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          v[i] = ex2(fmaf(v[i], sl2e, -mref));
          rs += v[i];
        }
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          v[i] = (i < nvalid) ? ex2(fmaf(v[i], sl2e, -mref)) : 0.f;
          rs += v[i];
        }
      }
      {
        uint32_t pw[32];  // P as bf16 pairs, key 2c in the low half of column c
#pragma unroll
        for (int c2 = 0; c2 < 32; ++c2) pw[c2] = pack_bf16(v[2 * c2], v[2 * c2 + 1]);
        tmem_st32(t_s, pw);  // over S_j, already read into registers
      }
      l += rs;
      tc_fence_before();
      mbar_arrive_cta(&p_full[g]);
    }
    // The stream's last PV; then stream 1 hands (m, l) over in shared memory
    // and stream 0 merges: O = (O_0 2^(m_0 - M) + O_1 2^(m_1 - M)) /
    // (l_0 2^(m_0 - M) + l_1 2^(m_1 - M)), M = max(m_0, m_1).
    const int nt = (ntiles - g + 1) / 2;  // tiles of this stream
    if (ok && nt > 0) ok = mbar_wait(&pv_full[g], (nt - 1) & 1, a.status, kStatusTimeoutAccum, abort_flag);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    if (g == 1) {
      xch[r] = nt > 0 ? mref : -INFINITY;
      xch[kQ + r] = l;
      xch[2 * kQ + r] = ok ? 1.f : 0.f;
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");  // both streams, every path
    // (warp-uniform: stream 1's flag is the same for the 32 rows of a quadrant)
    const bool has1 = ntiles > 1;
    if (g == 0 && __all_sync(0xffffffffu, ok && xch[2 * kQ + r] != 0.f)) {
      const float m1 = xch[r], l1 = xch[kQ + r];
      const float M = has1 ? fmaxf(mref, m1) : mref;
      const float f0 = ex2(mref - M), f1 = has1 ? ex2(m1 - M) : 0.f;
      const float den = l * f0 + l1 * f1;
      const float inv = 1.0f / den;
      const int qi = q0 + r;
      uint4* dst = reinterpret_cast<uint4*>(a.out + ((size_t)b * a.Lq + qi) * (a.H * kDh) + h * kDh);
#pragma unroll
      for (int half = 0; half < 2; ++half) {  // 32 channels at a time (registers)
        float o0[32];
        tmem_ld32(t_o + 32 * half, o0);
        if (has1) {
          float o1[32];
          tmem_ld32(t_lane + 128 + kDh + 32 * half, o1);
#pragma unroll
          for (int i = 0; i < 32; ++i) o0[i] = o0[i] * f0 + o1[i] * f1;
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o0[i] *= f0;
        }
        if (qi < a.Lq) {
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            uint4 w;
            w.x = pack_bf16(o0[8 * jj + 0] * inv, o0[8 * jj + 1] * inv);
            w.y = pack_bf16(o0[8 * jj + 2] * inv, o0[8 * jj + 3] * inv);
            w.z = pack_bf16(o0[8 * jj + 4] * inv, o0[8 * jj + 5] * inv);
            w.w = pack_bf16(o0[8 * jj + 6] * inv, o0[8 * jj + 7] * inv);
            dst[4 * half + jj] = w;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) {
      for (int g = 0; g < 2; ++g) {
        const int nt = (ntiles - g + 1) / 2;
        if (nt > 0) mbar_wait(&pv_full[g], (nt - 1) & 1, a.status, kStatusTimeoutDrain, nullptr);
      }
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  WAM_KT_END(attn, 1u);
}

}  // namespace

cudaError_t prepare_attention_tc() {
  return cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
}

cudaError_t launch_attention_tc(const AttnTc& t, cudaStream_t s) {
  if (t.Lq < 1 || t.Lk < 1) return cudaErrorInvalidValue;
  AttnTcK k;
  k.H = t.H;
  k.Lq = t.Lq;
  k.Lk = t.Lk;
  k.B = t.B;
  k.zq0 = t.zq0;
  k.zk0 = t.zk0;
  k.zv0 = t.zv0;
  k.out = reinterpret_cast<__nv_bfloat16*>(t.out);
  k.status = t.status;
  dim3 grid((t.Lq + kQ - 1) / kQ, t.H, t.B);
  return launch_k(attn_tc_kernel, grid, dim3(kThreads), kSmem, s, *t.map_q, *t.map_k, *t.map_v, k);
}

}  // namespace wam
