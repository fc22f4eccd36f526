// Allocation-free variant of the split-KV joint attention.
//
// Some callers cannot let a library allocate device memory while they run:
// a robot-control loop that must not call cudaMalloc after start-up (the
// call can synchronise the device and its latency is unbounded), or a
// process whose device memory budget is owned by another allocator.  For
// them, wam_op_attention_noalloc runs the same split-KV attention kernel as
// wam_op_attention, but its scratch -- the per-split partial outputs, row
// maxima and row sums, and the per-(sample, head) integer tickets that elect
// the combining CTA -- lives in the file-scope array below instead of in
// memory the library allocates.
//
// The array is part of the library's device image: every GPU that loads the
// library holds it (kScratchBytes) until the process exits.  All calls share
// it and it keeps the last call's contents, so calls that overlap on the GPU
// (on different streams, or from different threads) race on it.
#include <cstring>
#include <mutex>

#include "../../include/wam.h"
#include "kernels.h"

namespace {

constexpr size_t kScratchFloats = size_t(2) << 20;  // 8 MiB of partial outputs
constexpr int kTicketInts = 1024;                    // one per (sample, head)
constexpr size_t kScratchBytes = kScratchFloats * 4 + kTicketInts * 4;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of g_scratch on `dev` (which must be current).  Host code may
// not pass g_scratch itself to a kernel: on the host that name is a stand-in,
// not a device address.
cudaError_t scratch_address(int dev, void** out) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return e;
    // the split kernel's shared-memory limit is a per-device setting too
    if ((e = wam::prepare_attention_bf16()) != cudaSuccess) return e;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" wam_status wam_op_attention_noalloc(const void* q, const void* k, const void* v, void* out, int B, int H,
                                               int Lq, int Lk, int Lcache, int splits, void* stream) {
  if (!q || !k || !v || !out || B < 1 || H < 1 || Lq < 1 || Lq > 64 || Lk < 1 || Lk > Lcache || splits < 2)
    return WAM_ERR_INVALID_ARG;
  // Same split rule as the kernel's launcher: key blocks of a multiple of 64,
  // empty trailing splits dropped.
  int kps = (Lk + splits - 1) / splits;
  kps = (kps + 63) / 64 * 64;
  const int used = (Lk + kps - 1) / kps;
  if (used > 32) return WAM_ERR_UNSUPPORTED;  // the combine holds at most 32 splits
  const size_t need = wam::attention_ws_floats(B, H, 64, Lq, used);
  if (need > kScratchFloats || (size_t)B * H > (size_t)kTicketInts) return WAM_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return WAM_ERR_CUDA;
  void* base = nullptr;
  if (scratch_address(dev, &base) != cudaSuccess) return WAM_ERR_CUDA;
  float* ws = static_cast<float*>(base);
  int* tickets = reinterpret_cast<int*>(static_cast<unsigned char*>(base) + kScratchFloats * 4);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The kernel leaves its tickets at zero, but a previous call that did not
  // finish (an error on the stream) could leave them set: clear them first.
  if (cudaMemsetAsync(tickets, 0, (size_t)B * H * sizeof(int), s) != cudaSuccess) return WAM_ERR_CUDA;
  wam::AttnArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.out = out;
  a.B = B;
  a.H = H;
  a.Dh = 64;
  a.Lq = Lq;
  a.Lk = Lk;
  a.Lcache = Lcache;
  a.splits = splits;
  a.ws = ws;
  a.tickets = tickets;
  return wam::launch_attention_bf16(a, s) == cudaSuccess ? WAM_OK : WAM_ERR_CUDA;
}
