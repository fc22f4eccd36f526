// Video-query attention on the 5th-generation tensor cores (tcgen05).
//
// softmax(Q K^T / sqrt(64)) V for one (sample, head) and 128 queries per CTA,
// over keys [0, Lk) of the per-block cache (the video expert's own keys;
// RealtimeWAM summary page, 前置知识 "Mixture-of-Transformers": video queries
// see video keys only).
//
// Flash attention over 64-key tiles.  Two softmax warpgroups take the tiles
// in turn (g = j & 1), so two tiles are in flight; every tile has its own S and
// P buffers in tensor memory and all accumulate into one O:
//   S_j  = Q K_j^T      tcgen05.mma M=128 N=64 K=64, fp32 into TMEM S_g
//   P_j  = exp2(S_j log2e / 8 - m_j)   thread = query row, bf16 pairs into
//          TMEM P_g (separate columns, so S_{j+2} may overwrite S_g as soon as
//          S_j has been read, before PV_j runs)
//   O   += P_j V_j      tcgen05.mma M=128 N=64 K=64 accumulating in TMEM, P as
//          the A operand straight from TMEM, V as the MN-major B operand from
//          shared memory (the cache rows are [key][64 channels])
// The reference maximum m_j of a row is a chain through the tiles: m_j =
// m_{j-1} unless the tile's maximum exceeds it by more than 2^8, then the
// tile's maximum.  Warpgroup g takes m_{j-1} from the other one through shared
// memory (an mbarrier per tile parity) and publishes m_j as soon as it has the
// tile's maximum, before its exponentials.  A raised m (rare) rescales O once
// PV_{j-1} is complete and before PV_j is released; each warpgroup keeps its
// own row sum, brought to the final m at the end.  This is exact softmax
// arithmetic with a stale maximum (P <= 256).
// The S and PV products are issued by two threads (warps 1 and 2): one issue
// of an M=128 N=64 product costs about as long as it runs, so one thread
// issuing both would set the pace.  K and V tiles come by TMA through two
// 4-stage rings: a K stage is refilled as soon as its S product has run, so
// the K loads run ahead of the PV chain.
//
// Warp roles (384 threads): warp 0 TMA producer of Q and K, warp 1 TMEM owner
// + S issuer, warp 2 PV issuer, warp 3 TMA producer of V, warps 4..11 softmax: warpgroup
// (w-4)/4 takes tiles of its parity, warp w reads TMEM lanes 32*(w%4)..+31
// (its 32 query rows); at the end warpgroup g writes O's channels 32g..+31.
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
constexpr int kThreads = 384;              // producer, S issuer, PV issuer, idle, two softmax warpgroups
constexpr int kWG = 128;                   // threads of one softmax warpgroup
constexpr int kTmemCols = 256;
constexpr int kColS = 0;                   // S_0 [0, 64), S_1 [64, 128)
constexpr int kColO = 128;                 // O [128, 192)
constexpr int kColP = 192;                 // P_0 [192, 224), P_1 [224, 256) (bf16 pairs)
constexpr float kRescale = 8.0f;           // log2 headroom of the stale row maximum
constexpr int kXBytes = 2 * kQ * 4;        // m_j per row [tile parity][row]; the row sums at the end
constexpr int kBarBytes = 256;
// Two CTAs per SM: 2 x (82 KB + barriers + 1 KB reserved) <= 228 KB.
constexpr int kSmem = kQBytes + kStagesKV * 2 * kKVBytes + kXBytes + kBarBytes;

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

// 32 lanes x 32 consecutive 32-bit columns into r, without the wait: the
// registers are valid only after tmem_wait_ld64 below.
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      :
        "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// Waits for this thread's TMEM loads; the 64 registers are operands, so no
// use of them can be scheduled before the wait.
__device__ __forceinline__ void tmem_wait_ld64(uint32_t (&r)[64]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
      :
        "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
        "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
        "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
        "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31]),
        "+r"(r[32]), "+r"(r[33]), "+r"(r[34]), "+r"(r[35]), "+r"(r[36]), "+r"(r[37]), "+r"(r[38]), "+r"(r[39]),
        "+r"(r[40]), "+r"(r[41]), "+r"(r[42]), "+r"(r[43]), "+r"(r[44]), "+r"(r[45]), "+r"(r[46]), "+r"(r[47]),
        "+r"(r[48]), "+r"(r[49]), "+r"(r[50]), "+r"(r[51]), "+r"(r[52]), "+r"(r[53]), "+r"(r[54]), "+r"(r[55]),
        "+r"(r[56]), "+r"(r[57]), "+r"(r[58]), "+r"(r[59]), "+r"(r[60]), "+r"(r[61]), "+r"(r[62]), "+r"(r[63])
      :
      : "memory");
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

#ifdef WAM_ATTN_TIMELINE
// Diagnostic build only: %clock64 per key tile of the first four CTAs (head 0,
// sample 0) of the last launch.  Events: [j][0] S_j issued, [j][1] P_j seen by
// the PV issuer, [j][2] PV_j issued, then lane 0 of softmax quadrant 0: [j][3]
// S_j ready, [j][4] S_j read and its maximum taken, [j][5] exponentials done,
// [j][6] P_j stored, [j][7] S buffer free for S_j (S issuer); row 39: start, dependent-launch wait done, loop end,
// output written; row 38[0] the SM.
__device__ long long g_attn_tl[4][40][8];
// [cta][tile][quadrant][0: S_j in registers, 1: P_j released] (lane 0 of each quadrant)
__device__ long long g_attn_tlq[4][40][4][2];
#define ATLQ(j, q, e) \
  do { if (ATL_ON && (j) < 40 && lane == 0) g_attn_tlq[blockIdx.x][(j)][(q)][(e)] = clock64(); } while (0)
#define ATL_ON (blockIdx.y == 0 && blockIdx.z == 0 && blockIdx.x < 4)
#define ATL(j, e) \
  do { if (ATL_ON && (j) < 40) g_attn_tl[blockIdx.x][(j)][(e)] = clock64(); } while (0)
#else
#define ATL(j, e) do { } while (0)
#define ATLQ(j, q, e) do { } while (0)
#endif
namespace {

struct AttnTcK {
  int H, Lq, Lk, B;
  int zq0, zk0, zv0;  // z (matrix) index of (b=0, h=0) in the Q / K / V maps
  __nv_bfloat16* out;  // [B*Lq, H*64]
  unsigned* status;
};

// 32 lanes x 16 consecutive 32-bit columns from registers, one wait.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 32 fp32 values of this thread's TMEM lane back into 32 consecutive columns.
__device__ __forceinline__ void tmem_st32f(uint32_t taddr, const float (&v)[32]) {
  uint32_t r[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(v[i]);
  tmem_st32(taddr, r);
}

__global__ void __launch_bounds__(kThreads, 2)
    attn_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v, const AttnTcK a) {
  WAM_KT_BEGIN;
#ifdef WAM_ATTN_TIMELINE
  if (threadIdx.x == 0) {
    ATL(39, 0);
    unsigned sm;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
    if (ATL_ON) g_attn_tl[blockIdx.x][38][0] = sm;
  }
#endif
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
  float* xm = reinterpret_cast<float*>(sV + kStagesKV * kKVBytes);  // [2][128]
  uint64_t* bar = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(xm) + kXBytes);
  uint64_t* q_full = bar + 0;
  uint64_t* k_full = bar + 1;    // [4] K ring (refilled once S_j has read K_j)
  uint64_t* k_empty = bar + 5;   // [4]
  uint64_t* v_full = bar + 9;    // [4] V ring (refilled once PV_j has read V_j)
  uint64_t* v_empty = bar + 13;  // [4]
  uint64_t* s_full = bar + 17;   // [2] S_b written (S issuer -> softmax)
  uint64_t* s_free = bar + 19;   // [2] S_b read (softmax -> S issuer)
  uint64_t* p_full = bar + 21;   // [2] P_b written (softmax -> PV issuer)
  uint64_t* pv_done = bar + 23;  // [2] PV of tile j complete, j & 1 = b (PV issuer -> softmax)
  uint64_t* m_ready = bar + 25;  // [2] m_j of every row published (softmax g -> softmax 1 - g)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 27);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* issued = reinterpret_cast<int*>(tmem_slot + 2);  // [0] S tiles issued, [1] PV tiles issued

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * kQ, h = blockIdx.y, b = blockIdx.z;
  const int bh = b * a.H + h;
  const int ntiles = (a.Lk + kKT - 1) / kKT;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStagesKV; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], kWG);
      mbar_init(&p_full[i], kWG);
      mbar_init(&pv_done[i], 1);
      mbar_init(&m_ready[i], kWG);
    }
    *abort_flag = 0;
    issued[0] = 0;
    issued[1] = 0;
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

  if (warp == 0 || warp == 3) {
    // TMA producers: warp 0 loads Q and the K ring, warp 3 the V ring
    if (lane == 0) {
      pdl_wait();
      const bool is_k = warp == 0;
      if (is_k) {
        WAM_KT_WAITED();
        mbar_arrive_expect_tx(q_full, kQBytes);
        tma_load_3d(sQ, &map_q, q_full, 0, q0, a.zq0 + bh);
      }
      uint64_t* full = is_k ? k_full : v_full;
      uint64_t* empty = is_k ? k_empty : v_empty;
      uint8_t* ring = is_k ? sK : sV;
      const CUtensorMap* map = is_k ? &map_k : &map_v;
      const int z = (is_k ? a.zk0 : a.zv0) + bh;
      int nload = 0;
      for (int j = 0; j < ntiles; ++j) {
        const int s = j % kStagesKV;
        if (j >= kStagesKV &&
            !mbar_wait(&empty[s], ((j / kStagesKV) - 1) & 1, a.status, kStatusTimeoutTmaEmpty, abort_flag))
          break;
        mbar_arrive_expect_tx(&full[s], kKVBytes);
        tma_load_3d(ring + s * kKVBytes, map, &full[s], 0, j * kKT, z);
        nload = j + 1;
      }
      if (is_k) mbar_wait(q_full, 0, a.status, kStatusTimeoutDrain, nullptr);
      for (int j = max(0, nload - kStagesKV); j < nload; ++j)
        mbar_wait(&full[j % kStagesKV], (j / kStagesKV) & 1, a.status, kStatusTimeoutDrain, nullptr);
    }
  } else if (warp == 1) {
    // S issuer: S_j into S_{j & 1} once the softmax has read S_{j-2}
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kQ, kKT);
      const uint32_t aq = smem_u32(sQ);
      bool ok = mbar_wait(q_full, 0, a.status, kStatusTimeoutTmaFull, abort_flag);
      for (int j = 0; j < ntiles && ok; ++j) {
        const int bb = j & 1, s = j % kStagesKV;
        if (j >= 2 && !mbar_wait(&s_free[bb], ((j - 2) >> 1) & 1, a.status, kStatusTimeoutAccum, abort_flag)) break;
        ATL(j, 7);
        if (!mbar_wait(&k_full[s], (j / kStagesKV) & 1, a.status, kStatusTimeoutTmaFull, abort_flag)) break;
        tc_fence_after();
        const uint32_t ak = smem_u32(sK + s * kKVBytes);
#pragma unroll
        for (int kk = 0; kk < kDh / 16; ++kk)
          tc_mma_bf16(tmem + kColS + bb * kKT, smem_desc_k128(aq + kk * 32), smem_desc_k128(ak + kk * 32), idesc_s,
                      kk > 0 ? 1u : 0u);
        tc_commit(&s_full[bb]);
        tc_commit(&k_empty[s]);  // K_j is read once S_j completes
        issued[0] = j + 1;
        ATL(j, 0);
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // PV issuer: O += P_j V_j once the softmax has stored P_j
    if (lane == 0) {
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kQ, kDh) | (1u << 16);  // B (V) is MN-major
      for (int j = 0; j < ntiles; ++j) {
        const int bb = j & 1, s = j % kStagesKV;
        if (!mbar_wait(&p_full[bb], (j >> 1) & 1, a.status, kStatusTimeoutAccum, abort_flag)) break;
        if (!mbar_wait(&v_full[s], (j / kStagesKV) & 1, a.status, kStatusTimeoutTmaFull, abort_flag)) break;
        ATL(j, 1);
        tc_fence_after();
        const uint32_t av = smem_u32(sV + s * kKVBytes);
#pragma unroll
        for (int kk = 0; kk < kKT / 16; ++kk)  // 16 keys (8 columns of P) a step
          tc_mma_bf16_ts(tmem + kColO, tmem + kColP + bb * 32 + kk * 8, smem_desc_mn128(av + kk * 16 * 128),
                         idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&pv_done[bb]);
        tc_commit(&v_empty[s]);  // V_j is read once PV_j completes
        issued[1] = j + 1;
        ATL(j, 2);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------ softmax warps
    pdl_wait();
    const int quad = warp & 3;
    const int g = (warp - 4) >> 2;   // tiles g, g + 2, ...; O channels 32g..+31 at the end
    const int r = quad * 32 + lane;  // query row within the tile
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t t_s = t_lane + kColS + g * kKT, t_p = t_lane + kColP + g * 32, t_o = t_lane + kColO;
#ifdef WAM_ATTN_TIMELINE
    const bool tl_me = quad == 0 && lane == 0;
    if (tl_me && g == 0) ATL(39, 1);
#define ATLS(j, e) do { if (tl_me) ATL(j, e); } while (0)
#else
#define ATLS(j, e) do { } while (0)
#endif
    const float sl2e = 1.4426950408889634f * 0.125f;  // log2(e) / sqrt(64)
    float muse = -INFINITY, l = 0.f;  // m of this warpgroup's last tile, its row sum in those units
    bool ok = true;                   // warp-uniform
    for (int j = g; j < ntiles && ok; j += 2) {
      const int t = j >> 1;  // this warpgroup's tile count
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[g], t & 1, a.status, kStatusTimeoutAccum, abort_flag));
      if (!ok) break;
      ATLS(j, 3);
      tc_fence_after();
      const int nvalid = min(kKT, a.Lk - j * kKT);  // keys of this tile inside [0, Lk) (>= 1)
      // S_j into registers; S_g is then free
      float v[64];
      {
        uint32_t rr[64];
        tmem_ld32_async(t_s, rr);
        tmem_ld32_async(t_s + 32, rr + 32);
        tmem_wait_ld64(rr);
#pragma unroll
        for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(rr[i]);
      }
      tc_fence_before();
      mbar_arrive_cta(&s_free[g]);  // S_{j+2} may overwrite S_g
      ATLQ(j, quad, 0);
      if (nvalid < kKT) {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (i >= nvalid) v[i] = -INFINITY;  // exp2 gives 0 for them
      }
      float mx;
      {
        float m8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
          m8[k] = fmax3(fmax3(v[8 * k], v[8 * k + 1], v[8 * k + 2]), fmax3(v[8 * k + 3], v[8 * k + 4], v[8 * k + 5]),
                        fmaxf(v[8 * k + 6], v[8 * k + 7]));
        mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
      }
      const float mxs = mx * sl2e;
      // m_j from m_{j-1} (the other warpgroup's tile), published for tile j + 1
      float mprev = mxs, mj = mxs;
      if (j > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(&m_ready[(j - 1) & 1], ((j - 1) >> 1) & 1, a.status,
                                               kStatusTimeoutAccum, abort_flag));
        if (!ok) break;
        mprev = xm[((j - 1) & 1) * kQ + r];
        mj = mxs > mprev + kRescale ? mxs : mprev;
      }
      xm[(j & 1) * kQ + r] = mj;
      mbar_arrive_cta(&m_ready[j & 1]);
      ATLS(j, 4);
      if (muse != mj) {  // the row sum follows this warpgroup's m
        l *= ex2(muse - mj);  // 0 on the first tile (muse = -inf, l = 0)
        muse = mj;
      }
      // PV_{j-2} read P_g: it must be complete before P_j overwrites it
      if (j >= 2) {
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&pv_done[g], ((j - 2) >> 1) & 1, a.status, kStatusTimeoutAccum, abort_flag));
        if (!ok) break;
        tc_fence_after();
      }
      // P_j = exp2(S_j log2e / 8 - m_j) into P_g, 32 keys (16 columns) at a time
      float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pw[16];  // key 2c in the low half of column c
#pragma unroll
        for (int c2 = 0; c2 < 16; ++c2) {
          const float p0 = ex2(fmaf(v[32 * half + 2 * c2], sl2e, -mj));
          const float p1 = ex2(fmaf(v[32 * half + 2 * c2 + 1], sl2e, -mj));
          s4[(2 * c2) & 3] += p0;
          s4[(2 * c2 + 1) & 3] += p1;
          pw[c2] = pack_bf16(p0, p1);
        }
        tmem_st16(t_p + 16 * half, pw);
      }
      l += (s4[0] + s4[1]) + (s4[2] + s4[3]);
      ATLS(j, 5);
      // A raised m: O (PV_0 .. PV_{j-1}, in units of m_{j-1}) is rescaled
      // before PV_j is released
      const bool need = j > 0 && mj != mprev;
      if (__any_sync(0xffffffffu, need)) {  // tcgen05.ld / st are warp-wide
        ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, a.status,
                                               kStatusTimeoutAccum, abort_flag));
        if (!ok) break;
        tc_fence_after();
        const float alpha = need ? ex2(mprev - mj) : 1.f;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          float o[32];
          tmem_ld32(t_o + 32 * half, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32f(t_o + 32 * half, o);
        }
        tc_fence_before();
      }
      mbar_arrive_cta(&p_full[g]);
      ATLS(j, 6);
      ATLQ(j, quad, 1);
    }
    // The last PV and the last m; both row sums in units of that m; then
    // O / (l_0 + l_1) into the output rows, channels 32g..+31 by warpgroup g.
    const int n1 = ntiles - 1;
    ok = ok && __all_sync(0xffffffffu, mbar_wait(&pv_done[n1 & 1], (n1 >> 1) & 1, a.status, kStatusTimeoutAccum,
                                                 abort_flag));
    ok = ok && __all_sync(0xffffffffu, mbar_wait(&m_ready[n1 & 1], (n1 >> 1) & 1, a.status, kStatusTimeoutAccum,
                                                 abort_flag));
    tc_fence_after();
    ATLS(39, 2);
    const float mfin = ok ? xm[(n1 & 1) * kQ + r] : 0.f;
    if (ok && muse != mfin) l *= ex2(muse - mfin);  // 0 for a warpgroup without tiles
    asm volatile("bar.sync 1, 256;" ::: "memory");  // every m read; both warpgroups, every path
    xm[g * kQ + r] = l;
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (ok) {
      const float inv = 1.0f / (xm[r] + xm[kQ + r]);
      const int qi = q0 + r;
      float o[32];
      tmem_ld32(t_o + 32 * g, o);
      if (qi < a.Lq) {
        uint4* dst = reinterpret_cast<uint4*>(a.out + ((size_t)b * a.Lq + qi) * (a.H * kDh) + h * kDh + 32 * g);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          uint4 w;
          w.x = pack_bf16(o[8 * jj + 0] * inv, o[8 * jj + 1] * inv);
          w.y = pack_bf16(o[8 * jj + 2] * inv, o[8 * jj + 3] * inv);
          w.z = pack_bf16(o[8 * jj + 4] * inv, o[8 * jj + 5] * inv);
          w.w = pack_bf16(o[8 * jj + 6] * inv, o[8 * jj + 7] * inv);
          dst[jj] = w;
        }
      }
      ATLS(39, 3);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // Drain: every issued product complete before TMEM is released (only
    // waits on error paths; on success the softmax has seen them all).
    if (lane == 0) {
      const int ns = issued[0], npv = issued[1];
      if (ns > 0) mbar_wait(&s_full[(ns - 1) & 1], ((ns - 1) >> 1) & 1, a.status, kStatusTimeoutDrain, nullptr);
      if (npv > 0) mbar_wait(&pv_done[(npv - 1) & 1], ((npv - 1) >> 1) & 1, a.status, kStatusTimeoutDrain, nullptr);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  WAM_KT_END(attn, 1u);
}

}  // namespace

#ifdef WAM_ATTN_TIMELINE
extern "C" int wam_debug_attn_timeline(long long* host) {
  int r = cudaMemcpyFromSymbol(host, g_attn_tl, sizeof(g_attn_tl)) == cudaSuccess ? 0 : -1;
  if (cudaMemcpyFromSymbol(host + 4 * 40 * 8, g_attn_tlq, sizeof(g_attn_tlq)) != cudaSuccess) r = -1;
  static long long zero[4 * 40 * 8];
  cudaMemcpyToSymbol(g_attn_tl, zero, sizeof(zero));
  cudaMemcpyToSymbol(g_attn_tlq, zero, sizeof(zero));
  return r;
}
#endif

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
