// monarch_attn_fwd_noalloc: the bf16 forward pass for callers that cannot
// allocate device memory (see include/monarch_attn.h).
//
// It runs the same kernels as monarch_attn_fwd for the same shape.  The
// one-CTA-per-head kernel needs no scratch; the tensor-core path keeps its
// scratch (aggregated queries, Kt, Y, entropies) in one file-scope static
// device array of kScratchBytes, which every device that loads this library
// holds until the process exits.  Host code never names the array as a
// device address: at the first call on each device, with that device
// current, cudaGetSymbolAddress() yields the address that the kernels get.
// The status word (bounded-wait timeouts) is the library's static one,
// which monarch_attn_check() reads and clears.
#include "monarch_attn.h"

#include <mutex>

#include "entry.cuh"
#include "small_head.cuh"
#include "tc_path.cuh"

namespace {

constexpr size_t kScratchBytes = (size_t)64 << 20;  // 64 MiB
constexpr int kMaxDevices = 64;

// Scratch shared by every call of the entry point on one device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
char* g_scratch[kMaxDevices];  // resolved address of g_noalloc_scratch per device

// Once per device, with that device current: the device address of the
// scratch array (resolving it loads this file's device code on the device,
// which commits the array).
int scratch_address(int dev, char** out) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
      cudaGetLastError();
      return MONARCH_ERR_CUDA;
    }
    g_scratch[dev] = static_cast<char*>(p);
  }
  *out = g_scratch[dev];
  return MONARCH_OK;
}

}  // namespace

extern "C" int monarch_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                                        int B, int H, int b1, int b2, int d, int T, int c1,
                                        int c2, cudaStream_t stream) {
  if (!q || !k || !v || !out) return MONARCH_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, (const void*)out})
    if (reinterpret_cast<uintptr_t>(ptr) & 15u) return MONARCH_ERR_INVALID_ARG;
  int st = monarch::validate_args(B, H, b1, b2, d, T, c1, c2);
  if (st != MONARCH_OK) return st;
  // only the kernels that take d = 64 or 128 run here; checked before any
  // size arithmetic on d
  if (d != 64 && d != 128) return MONARCH_ERR_UNSUPPORTED;
  const monarch::Problem pb = monarch::make_problem(B, H, b1, b2, d, T, c1, c2);
  const monarch::Bf16Kernels kind = monarch::choose_bf16_kernels(pb);
  if (kind == monarch::Bf16Kernels::kSimt) return MONARCH_ERR_UNSUPPORTED;
  if (kind == monarch::Bf16Kernels::kTensorCore && monarch::tc_workspace_bytes(pb) > kScratchBytes)
    return MONARCH_ERR_SCRATCH_LIMIT;
  const size_t io = (size_t)pb.G * b1 * b2 * d * 2;
  const char* o0 = static_cast<const char*>(out);
  for (const void* in : {q, k, v}) {
    const char* i0 = static_cast<const char*>(in);
    if (o0 < i0 + io && i0 < o0 + io) return MONARCH_ERR_INVALID_ARG;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return MONARCH_ERR_CUDA;
  int* status = nullptr;
  if ((st = monarch::device_status_word(dev, &status)) != MONARCH_OK) return st;
  int launches = 0;
  cudaError_t e;
  if (kind == monarch::Bf16Kernels::kSmallHead) {
    e = monarch::small_head_forward(
        static_cast<const monarch::bf16*>(q), static_cast<const monarch::bf16*>(k),
        static_cast<const monarch::bf16*>(v), static_cast<monarch::bf16*>(out), pb, stream,
        &launches);
  } else {
    char* scratch = nullptr;
    if ((st = scratch_address(dev, &scratch)) != MONARCH_OK) return st;
    e = monarch::tc_forward(static_cast<const monarch::bf16*>(q),
                            static_cast<const monarch::bf16*>(k),
                            static_cast<const monarch::bf16*>(v),
                            static_cast<monarch::bf16*>(out), pb, scratch, status, stream,
                            &launches);
  }
  return e == cudaSuccess ? MONARCH_OK : MONARCH_ERR_CUDA;
}
