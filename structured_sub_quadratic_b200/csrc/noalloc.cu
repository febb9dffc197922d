// monarch_attn_fwd_noalloc: the bf16 forward pass for callers that cannot
// allocate device memory (see include/monarch_attn.h).
//
// Its scratch (aggregated queries, Kt, Y, entropies) lives in one file-scope
// static device array of kScratchBytes, which every device that loads this
// library holds until the process exits.  Host code never names the array
// as a device address: at the first call on each device, with that device
// current, cudaGetSymbolAddress() yields the address that the kernels get.
#include "monarch_attn.h"

#include <math.h>

#include <mutex>

#include "tc_path.cuh"

namespace {

constexpr size_t kScratchBytes = (size_t)64 << 20;  // 64 MiB
constexpr int kMaxDevices = 64;

// Scratch shared by every call of the entry point on one device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];
// Status word of those calls: a bounded device wait that expired sets it.
static __device__ __align__(256) int g_noalloc_status[64];

struct DeviceScratch {
  char* scratch = nullptr;
  int* status = nullptr;
  bool ready = false;
};

std::mutex g_mu;
DeviceScratch g_dev[kMaxDevices];

// Once per device, with that device current: resolve the device addresses
// of the static arrays and clear the status word.
int setup_device(int dev, DeviceScratch* out) {
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceScratch& s = g_dev[dev];
  if (!s.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return MONARCH_ERR_CUDA;
    char* scratch = static_cast<char*>(p);
    if (cudaGetSymbolAddress(&p, g_noalloc_status) != cudaSuccess) return MONARCH_ERR_CUDA;
    int* status = static_cast<int*>(p);
    if (cudaMemset(status, 0, sizeof(int)) != cudaSuccess) return MONARCH_ERR_CUDA;
    s.scratch = scratch;
    s.status = status;
    s.ready = true;
  }
  *out = s;
  return MONARCH_OK;
}

}  // namespace

extern "C" int monarch_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                                        int B, int H, int b1, int b2, int d, int T, int c1,
                                        int c2, cudaStream_t stream) {
  if (!q || !k || !v || !out) return MONARCH_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, (const void*)out})
    if (reinterpret_cast<uintptr_t>(ptr) & 15u) return MONARCH_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || b1 < 1 || b2 < 1 || T < 0 || c1 < 1 || c1 > b1 || c2 < 1 || c2 > b2)
    return MONARCH_ERR_INVALID_ARG;
  if ((long long)B * H > (1LL << 30)) return MONARCH_ERR_INVALID_ARG;
  const size_t io = (size_t)B * H * b1 * b2 * d * 2;
  const char* o0 = static_cast<const char*>(out);
  for (const void* in : {q, k, v}) {
    const char* i0 = static_cast<const char*>(in);
    if (o0 < i0 + io && i0 < o0 + io) return MONARCH_ERR_INVALID_ARG;
  }
  monarch::Problem pb;
  pb.G = B * H;
  pb.b1 = b1;
  pb.b2 = b2;
  pb.d = d;
  pb.T = T;
  pb.c1 = c1;
  pb.c2 = c2;
  pb.sc = 1.0f / sqrtf((float)d);
  if (!monarch::tc_supports(pb)) return MONARCH_ERR_UNSUPPORTED;
  if (monarch::tc_workspace_bytes(pb) > kScratchBytes) return MONARCH_ERR_SCRATCH_LIMIT;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return MONARCH_ERR_CUDA;
  DeviceScratch s;
  const int st = setup_device(dev, &s);
  if (st != MONARCH_OK) return st;
  int launches = 0;
  const cudaError_t e = monarch::tc_forward(
      static_cast<const monarch::bf16*>(q), static_cast<const monarch::bf16*>(k),
      static_cast<const monarch::bf16*>(v), static_cast<monarch::bf16*>(out), pb, s.scratch,
      s.status, stream, &launches);
  return e == cudaSuccess ? MONARCH_OK : MONARCH_ERR_CUDA;
}
