// C ABI of the MonarchAttention forward pass (declared in include/monarch_attn.h).
//
// This file validates arguments, owns the per-device workspace cache and the
// device status word, and dispatches to the kernels: the one-CTA-per-head
// kernel for small untiled bf16 heads with T >= 2, the tcgen05 tensor-core
// path for the other bf16 shapes it supports, the SIMT path for everything
// else.  The video-layout entry point reorders tokens around a forward call.
#include "monarch_attn.h"

#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "bwd_kernels.cuh"
#include "entry.cuh"
#include "layout.cuh"
#include "simt_kernels.cuh"
#include "small_head.cuh"
#include "tc_path.cuh"

// Status word of every entry point on a device: a bounded device wait that
// expires sets it (no kernel traps).  A static device variable, so neither
// entry point allocates for it; each device that loads the library holds
// its own copy, zero at load time.
static __device__ __align__(256) int g_status_word;

namespace {

using monarch::Problem;

constexpr int kMaxDevices = 64;
constexpr size_t kAlign = 256;

struct DevBuf {
  void* ptr = nullptr;
  size_t bytes = 0;
};

std::mutex g_mu;                // workspace and status words
std::mutex g_stage_mu;          // held for a whole host-buffer call
std::mutex g_layout_mu;         // held for a whole video-layout call
std::mutex g_pad_mu;            // held for a whole padded call
DevBuf g_ws[kMaxDevices];      // kernel workspace
DevBuf g_stage[kMaxDevices];   // staging for the host-buffer entry point

// Copy pipeline of the host-buffer entry point, per device (guarded by
// g_stage_mu; created on first use, kept until the process exits): a
// host-to-device and a device-to-host copy stream, and the events that order
// them with the caller's stream, one pair per group of heads.
constexpr int kHostChunks = 12;
constexpr size_t kHostGroupBytes = (size_t)32 << 20;
struct HostPipe {
  bool ready = false;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t in[kHostChunks] = {}, comp[kHostChunks] = {};
};
HostPipe g_pipe[kMaxDevices];
DevBuf g_layout[kMaxDevices];  // reordered q, k, v and output of the video-layout entry point
DevBuf g_pad[kMaxDevices];     // padded q, k, v and output of the padded entry point
DevBuf g_bwd[kMaxDevices];     // workspace of the backward pass

// Raster index tables of the video layouts used so far, per device (uploaded
// once per (f, h, w, layout); guarded by g_layout_mu).
struct PermTable {
  int f, h, w, layout;
  int* dev_table;
};
std::vector<PermTable> g_tables[kMaxDevices];
int* g_status[kMaxDevices];    // resolved address of g_status_word on each device
thread_local int t_launches = 0;
thread_local char t_err[256] = "";

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

int record_cuda(cudaError_t e) {
  std::snprintf(t_err, sizeof(t_err), "CUDA error: %s", cudaGetErrorString(e));
  return MONARCH_ERR_CUDA;
}

bool mul_ok(size_t a, size_t b, size_t* out) {
  if (a != 0 && b > SIZE_MAX / a) return false;
  *out = a * b;
  return true;
}

bool aligned16(const void* p) { return p != nullptr && ((uintptr_t)p & 15u) == 0; }

// Workspace of one call: none for the one-CTA-per-head kernel (small untiled
// heads with T >= 2, every step kept on chip), the tensor-core path's if it
// takes the shape, else the SIMT path's (fp32 pieces, each 256-byte aligned).
struct Plan {
  bool small = false;
  bool tc = false;
  size_t bytes = 0;
  monarch::SimtWorkspaceSizes simt{};
};

Plan make_plan(const Problem& pb, int dtype) {
  Plan pl;
  if (dtype == MONARCH_DTYPE_BF16) {
    switch (monarch::choose_bf16_kernels(pb)) {
      case monarch::Bf16Kernels::kSmallHead:
        pl.small = true;
        return pl;
      case monarch::Bf16Kernels::kTensorCore:
        pl.tc = true;
        pl.bytes = monarch::tc_workspace_bytes(pb);
        return pl;
      case monarch::Bf16Kernels::kSimt:
        break;
    }
  }
  pl.simt = monarch::simt_workspace_sizes(pb);
  const size_t* f = &pl.simt.qt0;
  for (int t = 0; t < 7; ++t) pl.bytes += align_up(f[t] * sizeof(float));
  return pl;
}

monarch::SimtWorkspace carve_simt(const Plan& pl, char* base) {
  monarch::SimtWorkspace ws;
  void* dst[7];
  const size_t* f = &pl.simt.qt0;
  size_t off = 0;
  for (int t = 0; t < 7; ++t) {
    dst[t] = f[t] ? static_cast<void*>(base + off) : nullptr;
    off += align_up(f[t] * sizeof(float));
  }
  ws.qt0 = static_cast<float*>(dst[0]);
  ws.qt = static_cast<float*>(dst[1]);
  ws.kt = dst[2];
  ws.y = dst[3];
  ws.hs = static_cast<float*>(dst[4]);
  ws.lse = static_cast<float*>(dst[5]);
  ws.ybar = static_cast<float*>(dst[6]);
  return ws;
}

int current_device(int* dev) {
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return record_cuda(e);
  if (*dev < 0 || *dev >= kMaxDevices) return MONARCH_ERR_UNSUPPORTED;
  return MONARCH_OK;
}

// Host-side fault injection: with MONARCH_ATTN_FAIL_ALLOC=1 in the
// environment every workspace or staging allocation the library attempts
// fails as if cudaMalloc had run out of memory (no device call is made).
bool alloc_failure_injected() {
  const char* e = std::getenv("MONARCH_ATTN_FAIL_ALLOC");
  return e != nullptr && e[0] == '1';
}

// Grow-only cached device buffer.  cudaFree synchronises the device, so a
// buffer still used by an earlier call is never freed under it.
int ensure(DevBuf& b, size_t bytes) {
  if (bytes <= b.bytes) return MONARCH_OK;
  if (alloc_failure_injected()) {
    std::snprintf(t_err, sizeof(t_err),
                  "workspace allocation of %zu bytes failed (injected by MONARCH_ATTN_FAIL_ALLOC)",
                  bytes);
    return MONARCH_ERR_NO_MEMORY;
  }
  if (b.ptr) {
    cudaError_t e = cudaFree(b.ptr);
    b.ptr = nullptr;
    b.bytes = 0;
    if (e != cudaSuccess) return record_cuda(e);
  }
  cudaError_t e = cudaMalloc(&b.ptr, bytes);
  if (e != cudaSuccess) {
    b.ptr = nullptr;
    cudaGetLastError();
    std::snprintf(t_err, sizeof(t_err), "workspace allocation of %zu bytes failed: %s", bytes,
                  cudaGetErrorString(e));
    return MONARCH_ERR_NO_MEMORY;
  }
  b.bytes = bytes;
  return MONARCH_OK;
}

// Device address of g_status_word on `dev` (current), resolved once.  g_mu held.
int status_word_locked(int dev, int** out) {
  if (!g_status[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_status_word);
    if (e != cudaSuccess) return record_cuda(e);
    g_status[dev] = static_cast<int*>(p);
  }
  *out = g_status[dev];
  return MONARCH_OK;
}

// real_lo, real_hi: the real tokens of the b1*b2 grid (padding; the default
// is every token).  q, k, v, out always hold whole grids here.
// init_units: the launch-shape hint of Problem (a call split into groups of
// heads passes the whole call's unit count).
template <typename TIn>
int forward_device(const TIn* q, const TIn* k, const TIn* v, TIn* out, int B, int H, int b1,
                   int b2, int d, int T, int c1, int c2, cudaStream_t stream, int dtype,
                   int real_lo = 0, int real_hi = -1, int tr = 0, long init_units = 0) {
  t_launches = 0;
  int st = monarch::validate_args(B, H, b1, b2, d, T, c1, c2);
  if (st != MONARCH_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return MONARCH_ERR_INVALID_ARG;
  Problem pb = monarch::make_problem(B, H, b1, b2, d, T, c1, c2);
  if (real_hi >= 0) {
    pb.real_lo = real_lo;
    pb.real_hi = real_hi;
  }
  pb.tr = tr;
  pb.init_units = init_units;
  const size_t bytes_io = (size_t)pb.G * b1 * b2 * d * sizeof(TIn);
  const char* o0 = reinterpret_cast<const char*>(out);
  for (const void* in : {(const void*)q, (const void*)k, (const void*)v}) {
    const char* i0 = reinterpret_cast<const char*>(in);
    if (o0 < i0 + bytes_io && i0 < o0 + bytes_io) return MONARCH_ERR_INVALID_ARG;
  }
  int dev;
  if ((st = current_device(&dev)) != MONARCH_OK) return st;
  const Plan pl = make_plan(pb, dtype);
  std::lock_guard<std::mutex> lock(g_mu);
  int* status = nullptr;
  if ((st = status_word_locked(dev, &status)) != MONARCH_OK) return st;
  if ((st = ensure(g_ws[dev], pl.bytes ? pl.bytes : kAlign)) != MONARCH_OK) return st;
  cudaError_t e;
  if (pl.small) {
    e = monarch::small_head_forward(reinterpret_cast<const monarch::bf16*>(q),
                                    reinterpret_cast<const monarch::bf16*>(k),
                                    reinterpret_cast<const monarch::bf16*>(v),
                                    reinterpret_cast<monarch::bf16*>(out), pb, stream, &t_launches);
  } else if (pl.tc) {
    e = monarch::tc_forward(reinterpret_cast<const monarch::bf16*>(q),
                            reinterpret_cast<const monarch::bf16*>(k),
                            reinterpret_cast<const monarch::bf16*>(v),
                            reinterpret_cast<monarch::bf16*>(out), pb,
                            static_cast<char*>(g_ws[dev].ptr), status, stream,
                            &t_launches);
  } else {
    const monarch::SimtWorkspace ws = carve_simt(pl, static_cast<char*>(g_ws[dev].ptr));
    e = monarch::simt_forward<TIn, float>(q, k, v, out, pb, ws, stream, &t_launches);
  }
  if (e != cudaSuccess) return record_cuda(e);
  return MONARCH_OK;
}

}  // namespace

namespace monarch {

int validate_args(int B, int H, int b1, int b2, int d, int T, int c1, int c2) {
  if (B < 1 || H < 1 || b1 < 1 || b2 < 1 || T < 0) return MONARCH_ERR_INVALID_ARG;
  if (c1 < 1 || c1 > b1 || c2 < 1 || c2 > b2) return MONARCH_ERR_INVALID_ARG;
  if (d < 1 || d > 256) return MONARCH_ERR_UNSUPPORTED;
  size_t n;
  if (!mul_ok((size_t)B, (size_t)H, &n) || !mul_ok(n, (size_t)b1, &n) ||
      !mul_ok(n, (size_t)b2, &n) || !mul_ok(n, (size_t)d, &n) || !mul_ok(n, (size_t)c1, &n) ||
      !mul_ok(n, (size_t)c2, &n) || n > ((size_t)1 << 40))
    return MONARCH_ERR_INVALID_ARG;
  if ((long long)B * H > (1LL << 30)) return MONARCH_ERR_INVALID_ARG;
  return MONARCH_OK;
}

Problem make_problem(int B, int H, int b1, int b2, int d, int T, int c1, int c2) {
  Problem pb;
  pb.G = B * H;
  pb.b1 = b1;
  pb.b2 = b2;
  pb.d = d;
  pb.T = T;
  pb.c1 = c1;
  pb.c2 = c2;
  pb.sc = 1.0f / sqrtf((float)d);
  pb.real_lo = 0;
  pb.real_hi = b1 * b2;
  pb.tr = 0;
  pb.init_units = 0;
  return pb;
}

Bf16Kernels choose_bf16_kernels(const Problem& pb) {
  // Small untiled heads with T >= 2 keep every step in one CTA (their later
  // steps would otherwise run on the SIMT kernels).
  if (pb.T >= 2 && small_head_supports(pb)) return Bf16Kernels::kSmallHead;
  if (tc_supports(pb)) return Bf16Kernels::kTensorCore;
  return Bf16Kernels::kSimt;
}

int device_status_word(int dev, int** out) {
  if (dev < 0 || dev >= kMaxDevices) return MONARCH_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  return status_word_locked(dev, out);
}

}  // namespace monarch

extern "C" {

int monarch_attn_fwd(const void* q, const void* k, const void* v, void* out, int B, int H,
                     int b1, int b2, int d, int T, int c1, int c2, cudaStream_t stream) {
  using monarch::bf16;
  return forward_device<bf16>(static_cast<const bf16*>(q), static_cast<const bf16*>(k),
                              static_cast<const bf16*>(v), static_cast<bf16*>(out), B, H, b1, b2,
                              d, T, c1, c2, stream, MONARCH_DTYPE_BF16);
}

int monarch_attn_fwd_f32(const float* q, const float* k, const float* v, float* out, int B,
                         int H, int b1, int b2, int d, int T, int c1, int c2,
                         cudaStream_t stream) {
  return forward_device<float>(q, k, v, out, B, H, b1, b2, d, T, c1, c2, stream,
                               MONARCH_DTYPE_F32);
}

int monarch_attn_fwd_host(int dtype, const void* q_host, const void* k_host, const void* v_host,
                          void* out_host, int B, int H, int b1, int b2, int d, int T, int c1,
                          int c2, cudaStream_t stream) {
  if (dtype != MONARCH_DTYPE_BF16 && dtype != MONARCH_DTYPE_F32) return MONARCH_ERR_INVALID_ARG;
  if (!q_host || !k_host || !v_host || !out_host) return MONARCH_ERR_INVALID_ARG;
  int st = monarch::validate_args(B, H, b1, b2, d, T, c1, c2);
  if (st != MONARCH_OK) return st;
  const size_t elt = dtype == MONARCH_DTYPE_BF16 ? 2 : 4;
  const size_t head_bytes = (size_t)b1 * b2 * d * elt;
  const long G = (long)B * H;
  const size_t n = (size_t)G * head_bytes;
  const size_t slot = align_up(n);
  int dev;
  if ((st = current_device(&dev)) != MONARCH_OK) return st;
  std::lock_guard<std::mutex> stage_lock(g_stage_mu);
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if ((st = ensure(g_stage[dev], 4 * slot)) != MONARCH_OK) return st;
  }
  HostPipe& pp = g_pipe[dev];
  cudaError_t e = cudaSuccess;
  if (!pp.ready) {
    if ((e = cudaStreamCreateWithFlags(&pp.h2d, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&pp.d2h, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&pp.start, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&pp.done, cudaEventDisableTiming)) != cudaSuccess)
      return record_cuda(e);
    for (int c = 0; c < kHostChunks; ++c)
      if ((e = cudaEventCreateWithFlags(&pp.in[c], cudaEventDisableTiming)) != cudaSuccess ||
          (e = cudaEventCreateWithFlags(&pp.comp[c], cudaEventDisableTiming)) != cudaSuccess)
        return record_cuda(e);
    pp.ready = true;
  }
  char* base = static_cast<char*>(g_stage[dev].ptr);
  char *dq = base, *dk = base + slot, *dv = base + 2 * slot, *dout = base + 3 * slot;
  // Heads are independent: groups of heads are copied in on pp.h2d, computed
  // on `stream` and copied out on pp.d2h, so that group c + 1's copy-in and
  // group c - 1's copy-out overlap group c's forward pass.  Each group runs
  // the kernels of the whole call (the launch-shape hint), so the output is
  // bit-identical to monarch_attn_fwd's.
  // groups of at least kHostGroupBytes of input (a smaller call's forward
  // pass is too short to hide copies behind, and each group adds copy and
  // launch overhead), at most kHostChunks
  const long groups = std::max(1L, std::min((long)kHostChunks, (long)(3 * n / kHostGroupBytes)));
  const long hc = (G + groups - 1) / groups;  // heads per group
  const int nc = (int)((G + hc - 1) / hc);
  const long init_units = G * c1 * b2;
  const auto* qh = static_cast<const char*>(q_host);
  const auto* kh = static_cast<const char*>(k_host);
  const auto* vh = static_cast<const char*>(v_host);
  auto* oh = static_cast<char*>(out_host);
  int launches = 0;
  // the copies start after the work already on `stream`
  if ((e = cudaEventRecord(pp.start, stream)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(pp.h2d, pp.start, 0)) != cudaSuccess)
    return record_cuda(e);
  for (int c = 0; c < nc && st == MONARCH_OK && e == cudaSuccess; ++c) {
    const long h0 = c * hc, hn = std::min(hc, G - h0);
    const size_t off = (size_t)h0 * head_bytes, bytes = (size_t)hn * head_bytes;
    if ((e = cudaMemcpyAsync(dq + off, qh + off, bytes, cudaMemcpyHostToDevice, pp.h2d)) !=
            cudaSuccess ||
        (e = cudaMemcpyAsync(dk + off, kh + off, bytes, cudaMemcpyHostToDevice, pp.h2d)) !=
            cudaSuccess ||
        (e = cudaMemcpyAsync(dv + off, vh + off, bytes, cudaMemcpyHostToDevice, pp.h2d)) !=
            cudaSuccess ||
        (e = cudaEventRecord(pp.in[c], pp.h2d)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(stream, pp.in[c], 0)) != cudaSuccess)
      break;
    st = dtype == MONARCH_DTYPE_BF16
             ? forward_device<monarch::bf16>(
                   reinterpret_cast<const monarch::bf16*>(dq + off),
                   reinterpret_cast<const monarch::bf16*>(dk + off),
                   reinterpret_cast<const monarch::bf16*>(dv + off),
                   reinterpret_cast<monarch::bf16*>(dout + off), 1, (int)hn, b1, b2, d, T, c1, c2,
                   stream, MONARCH_DTYPE_BF16, 0, -1, 0, init_units)
             : forward_device<float>(reinterpret_cast<const float*>(dq + off),
                                     reinterpret_cast<const float*>(dk + off),
                                     reinterpret_cast<const float*>(dv + off),
                                     reinterpret_cast<float*>(dout + off), 1, (int)hn, b1, b2, d,
                                     T, c1, c2, stream, MONARCH_DTYPE_F32, 0, -1, 0, init_units);
    launches += t_launches;
    if (st != MONARCH_OK) break;
    if ((e = cudaEventRecord(pp.comp[c], stream)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(pp.d2h, pp.comp[c], 0)) != cudaSuccess ||
        (e = cudaMemcpyAsync(oh + off, dout + off, bytes, cudaMemcpyDeviceToHost, pp.d2h)) !=
            cudaSuccess)
      break;
  }
  if (e == cudaSuccess && st == MONARCH_OK) {
    if ((e = cudaEventRecord(pp.done, pp.d2h)) == cudaSuccess)
      e = cudaStreamWaitEvent(stream, pp.done, 0);
  }
  t_launches = launches;
  if (e != cudaSuccess || st != MONARCH_OK) {
    // nothing may still read or write the caller's buffers after the return
    cudaStreamSynchronize(pp.h2d);
    cudaStreamSynchronize(pp.d2h);
    cudaStreamSynchronize(stream);
    return e != cudaSuccess ? record_cuda(e) : st;
  }
  return monarch_attn_check(stream);
}

int monarch_attn_fwd_video(int dtype, const void* q, const void* k, const void* v, void* out,
                           int B, int H, int f, int h, int w, int layout, int d, int T, int c1,
                           int c2, cudaStream_t stream) {
  if (dtype != MONARCH_DTYPE_BF16 && dtype != MONARCH_DTYPE_F32) return MONARCH_ERR_INVALID_ARG;
  if (layout < MONARCH_LAYOUT_FH_W || layout > MONARCH_LAYOUT_H_FW) return MONARCH_ERR_INVALID_ARG;
  if (f < 1 || h < 1 || w < 1 || (long long)f * h * w > (1LL << 30)) return MONARCH_ERR_INVALID_ARG;
  // axes in Monarch order (sizes, raster strides in tokens) and the row-group size b1
  const long hw = (long)h * w;
  monarch::VideoPerm vp;
  long b1 = 0;
  auto axes = [&](int s0, long t0, int s1, long t1, int s2, long t2, long rows) {
    vp.s[0] = s0; vp.t[0] = t0;
    vp.s[1] = s1; vp.t[1] = t1;
    vp.s[2] = s2; vp.t[2] = t2;
    b1 = rows;
  };
  switch (layout) {
    case MONARCH_LAYOUT_FH_W: axes(f, hw, h, w, w, 1, (long)f * h); break;
    case MONARCH_LAYOUT_W_FH: axes(w, 1, f, hw, h, w, w); break;
    case MONARCH_LAYOUT_F_HW: axes(f, hw, h, w, w, 1, f); break;
    case MONARCH_LAYOUT_HW_F: axes(h, w, w, 1, f, hw, hw); break;
    case MONARCH_LAYOUT_FW_H: axes(f, hw, w, 1, h, w, (long)f * w); break;
    default: axes(h, w, f, hw, w, 1, h); break;  // MONARCH_LAYOUT_H_FW
  }
  const int N = (int)((long)f * hw), rows = (int)b1, cols = N / rows;
  int st = monarch::validate_args(B, H, rows, cols, d, T, c1, c2);
  if (st != MONARCH_OK) return st;
  auto fwd = [&](const void* a, const void* b, const void* c, void* o) {
    return dtype == MONARCH_DTYPE_BF16
               ? monarch_attn_fwd(a, b, c, o, B, H, rows, cols, d, T, c1, c2, stream)
               : monarch_attn_fwd_f32(static_cast<const float*>(a), static_cast<const float*>(b),
                                      static_cast<const float*>(c), static_cast<float*>(o), B, H,
                                      rows, cols, d, T, c1, c2, stream);
  };
  if (layout == MONARCH_LAYOUT_FH_W || layout == MONARCH_LAYOUT_F_HW) return fwd(q, k, v, out);
  // (w,fh) and (hw,f): raster token i*b1 + l is the transpose of Monarch
  // order, which the tensor-core kernels read and write in place (no
  // gather, no scatter) when every kernel of the pass is a tensor-core one
  if (dtype == MONARCH_DTYPE_BF16 &&
      (layout == MONARCH_LAYOUT_W_FH || layout == MONARCH_LAYOUT_HW_F)) {
    Problem pt = monarch::make_problem(B, H, rows, cols, d, T, c1, c2);
    pt.tr = 1;
    if (monarch::choose_bf16_kernels(pt) == monarch::Bf16Kernels::kTensorCore &&
        monarch::tc_takes_transposed(pt))
      return forward_device<monarch::bf16>(
          static_cast<const monarch::bf16*>(q), static_cast<const monarch::bf16*>(k),
          static_cast<const monarch::bf16*>(v), static_cast<monarch::bf16*>(out), B, H, rows,
          cols, d, T, c1, c2, stream, MONARCH_DTYPE_BF16, 0, -1, 1);
  }
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return MONARCH_ERR_INVALID_ARG;
  const int row_bytes = d * (dtype == MONARCH_DTYPE_BF16 ? 2 : 4);
  const size_t slot = align_up((size_t)B * H * N * row_bytes);
  int dev;
  if ((st = current_device(&dev)) != MONARCH_OK) return st;
  std::lock_guard<std::mutex> layout_lock(g_layout_mu);
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if ((st = ensure(g_layout[dev], 4 * slot)) != MONARCH_OK) return st;
  }
  char* base = static_cast<char*>(g_layout[dev].ptr);
  char *dq = base, *dk = base + slot, *dv = base + 2 * slot, *dout = base + 3 * slot;
  const int* table = nullptr;
  for (const PermTable& t : g_tables[dev])
    if (t.f == f && t.h == h && t.w == w && t.layout == layout) table = t.dev_table;
  cudaError_t e;
  if (!table) {  // first use of this latent and layout on this device: build and upload
    std::vector<int> host(N);
    monarch::video_perm_table(vp, host.data());
    int* p = nullptr;
    if ((e = cudaMalloc(&p, sizeof(int) * N)) != cudaSuccess) return record_cuda(e);
    if ((e = cudaMemcpy(p, host.data(), sizeof(int) * N, cudaMemcpyHostToDevice)) !=
        cudaSuccess) {
      cudaFree(p);
      return record_cuda(e);
    }
    g_tables[dev].push_back({f, h, w, layout, p});
    table = p;
  }
  const long G = (long)B * H;
  int perm_launches = 0;
  const void* in_src[3] = {q, k, v};
  void* in_dst[3] = {dq, dk, dv};
  if ((e = monarch::permute_rows(in_src, in_dst, 3, table, G, N, row_bytes, true, stream,
                                 &perm_launches)) != cudaSuccess)
    return record_cuda(e);
  if ((st = fwd(dq, dk, dv, dout)) != MONARCH_OK) return st;
  const void* out_src[1] = {dout};
  void* out_dst[1] = {out};
  if ((e = monarch::permute_rows(out_src, out_dst, 1, table, G, N, row_bytes, false, stream,
                                 &perm_launches)) != cudaSuccess)
    return record_cuda(e);
  t_launches += perm_launches;
  return MONARCH_OK;
}

int monarch_attn_fwd_padded(int dtype, const void* q, const void* k, const void* v, void* out,
                            int B, int H, int n_real, int b1, int b2, int pad_front, int d, int T,
                            int c1, int c2, cudaStream_t stream) {
  t_launches = 0;
  if (dtype != MONARCH_DTYPE_BF16 && dtype != MONARCH_DTYPE_F32) return MONARCH_ERR_INVALID_ARG;
  if (pad_front != 0 && pad_front != 1) return MONARCH_ERR_INVALID_ARG;
  int st = monarch::validate_args(B, H, b1, b2, d, T, c1, c2);
  if (st != MONARCH_OK) return st;
  const int N = b1 * b2;
  if (n_real < 1 || n_real > N) return MONARCH_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return MONARCH_ERR_INVALID_ARG;
  using monarch::bf16;
  if (n_real == N)
    return dtype == MONARCH_DTYPE_BF16
               ? monarch_attn_fwd(q, k, v, out, B, H, b1, b2, d, T, c1, c2, stream)
               : monarch_attn_fwd_f32(static_cast<const float*>(q), static_cast<const float*>(k),
                                      static_cast<const float*>(v), static_cast<float*>(out), B,
                                      H, b1, b2, d, T, c1, c2, stream);
  const int real_lo = pad_front ? N - n_real : 0;
  Problem pb = monarch::make_problem(B, H, b1, b2, d, T, c1, c2);
  pb.real_lo = real_lo;
  pb.real_hi = real_lo + n_real;
  const int row_bytes = d * (dtype == MONARCH_DTYPE_BF16 ? 2 : 4);
  const size_t bytes_io = (size_t)pb.G * n_real * row_bytes;
  const char* o0 = static_cast<const char*>(out);
  for (const void* in : {q, k, v}) {
    const char* i0 = static_cast<const char*>(in);
    if (o0 < i0 + bytes_io && i0 < o0 + bytes_io) return MONARCH_ERR_INVALID_ARG;
  }
  int dev;
  if ((st = current_device(&dev)) != MONARCH_OK) return st;
  if (dtype == MONARCH_DTYPE_BF16 &&
      monarch::choose_bf16_kernels(pb) == monarch::Bf16Kernels::kSmallHead) {
    // small heads: the kernel reads and writes the real rows in place
    const cudaError_t e = monarch::small_head_forward(
        static_cast<const bf16*>(q), static_cast<const bf16*>(k), static_cast<const bf16*>(v),
        static_cast<bf16*>(out), pb, stream, &t_launches);
    return e == cudaSuccess ? MONARCH_OK : record_cuda(e);
  }
  // every other kernel works on whole grids: pad q, k, v into a cached
  // buffer, run the masked forward pass, copy the real output rows back
  const size_t slot = align_up((size_t)pb.G * N * row_bytes);
  std::lock_guard<std::mutex> pad_lock(g_pad_mu);
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if ((st = ensure(g_pad[dev], 4 * slot)) != MONARCH_OK) return st;
  }
  char* base = static_cast<char*>(g_pad[dev].ptr);
  char *dq = base, *dk = base + slot, *dv = base + 2 * slot, *dout = base + 3 * slot;
  int pad_launches = 0;
  const void* in_src[3] = {q, k, v};
  void* in_dst[3] = {dq, dk, dv};
  cudaError_t e = monarch::pad_rows(in_src, in_dst, 3, pb.G, N, n_real, real_lo, row_bytes, true,
                                    stream, &pad_launches);
  if (e != cudaSuccess) return record_cuda(e);
  st = dtype == MONARCH_DTYPE_BF16
           ? forward_device<bf16>(reinterpret_cast<const bf16*>(dq),
                                  reinterpret_cast<const bf16*>(dk),
                                  reinterpret_cast<const bf16*>(dv), reinterpret_cast<bf16*>(dout),
                                  B, H, b1, b2, d, T, c1, c2, stream, MONARCH_DTYPE_BF16,
                                  pb.real_lo, pb.real_hi)
           : forward_device<float>(reinterpret_cast<const float*>(dq),
                                   reinterpret_cast<const float*>(dk),
                                   reinterpret_cast<const float*>(dv),
                                   reinterpret_cast<float*>(dout), B, H, b1, b2, d, T, c1, c2,
                                   stream, MONARCH_DTYPE_F32, pb.real_lo, pb.real_hi);
  if (st != MONARCH_OK) return st;
  const void* out_src[1] = {dout};
  void* out_dst[1] = {out};
  e = monarch::pad_rows(out_src, out_dst, 1, pb.G, N, n_real, real_lo, row_bytes, false, stream,
                        &pad_launches);
  if (e != cudaSuccess) return record_cuda(e);
  t_launches += pad_launches;
  return MONARCH_OK;
}

int monarch_attn_bwd(int dtype, const void* q, const void* k, const void* v, const void* dout,
                     void* dq, void* dk, void* dv, int B, int H, int b1, int b2, int d, int T,
                     int c1, int c2, cudaStream_t stream) {
  t_launches = 0;
  if (dtype != MONARCH_DTYPE_BF16 && dtype != MONARCH_DTYPE_F32) return MONARCH_ERR_INVALID_ARG;
  int st = monarch::validate_args(B, H, b1, b2, d, T, c1, c2);
  if (st != MONARCH_OK) return st;
  if (T != 1) return MONARCH_ERR_UNSUPPORTED;
  for (const void* ptr : {q, k, v, dout, (const void*)dq, (const void*)dk, (const void*)dv})
    if (!aligned16(ptr)) return MONARCH_ERR_INVALID_ARG;
  const Problem pb = monarch::make_problem(B, H, b1, b2, d, T, c1, c2);
  const size_t bytes_io = (size_t)pb.G * b1 * b2 * d * (dtype == MONARCH_DTYPE_BF16 ? 2 : 4);
  const void* ins[4] = {q, k, v, dout};
  const void* outs[3] = {dq, dk, dv};
  for (const void* o : outs)
    for (const void* in : ins) {
      const char *o0 = static_cast<const char*>(o), *i0 = static_cast<const char*>(in);
      if (o0 < i0 + bytes_io && i0 < o0 + bytes_io) return MONARCH_ERR_INVALID_ARG;
    }
  for (int a = 0; a < 3; ++a)
    for (int b = a + 1; b < 3; ++b) {
      const char *x = static_cast<const char*>(outs[a]), *y = static_cast<const char*>(outs[b]);
      if (x < y + bytes_io && y < x + bytes_io) return MONARCH_ERR_INVALID_ARG;
    }
  int dev;
  if ((st = current_device(&dev)) != MONARCH_OK) return st;
  const monarch::BwdWorkspaceSizes sz = monarch::bwd_workspace_sizes(pb);
  const size_t* f = &sz.qt0;
  constexpr int kPieces = sizeof(sz) / sizeof(size_t);
  size_t total = 0;
  for (int t = 0; t < kPieces; ++t) total += align_up(f[t] * sizeof(float));
  std::lock_guard<std::mutex> lock(g_mu);
  if ((st = ensure(g_bwd[dev], total)) != MONARCH_OK) return st;
  int* status = nullptr;
  if ((st = status_word_locked(dev, &status)) != MONARCH_OK) return st;
  monarch::BwdWorkspace ws;
  float** dst = &ws.qt0;
  char* base = static_cast<char*>(g_bwd[dev].ptr);
  size_t off = 0;
  for (int t = 0; t < kPieces; ++t) {
    dst[t] = reinterpret_cast<float*>(base + off);
    off += align_up(f[t] * sizeof(float));
  }
  using monarch::bf16;
  const cudaError_t e =
      dtype == MONARCH_DTYPE_BF16
          ? monarch::bwd_forward_t1<bf16>(
                static_cast<const bf16*>(q), static_cast<const bf16*>(k),
                static_cast<const bf16*>(v), static_cast<const bf16*>(dout),
                static_cast<bf16*>(dq), static_cast<bf16*>(dk), static_cast<bf16*>(dv), pb, ws,
                status, stream, &t_launches)
          : monarch::bwd_forward_t1<float>(
                static_cast<const float*>(q), static_cast<const float*>(k),
                static_cast<const float*>(v), static_cast<const float*>(dout),
                static_cast<float*>(dq), static_cast<float*>(dk), static_cast<float*>(dv), pb, ws,
                status, stream, &t_launches);
  return e == cudaSuccess ? MONARCH_OK : record_cuda(e);
}

size_t monarch_attn_workspace_bytes(int B, int H, int b1, int b2, int d, int T, int c1, int c2,
                                    int dtype) {
  if (monarch::validate_args(B, H, b1, b2, d, T, c1, c2) != MONARCH_OK) return 0;
  if (dtype != MONARCH_DTYPE_BF16 && dtype != MONARCH_DTYPE_F32) return 0;
  return make_plan(monarch::make_problem(B, H, b1, b2, d, T, c1, c2), dtype).bytes;
}

void monarch_attn_release_workspace(void) {
  std::lock_guard<std::mutex> pad_lock(g_pad_mu);
  std::lock_guard<std::mutex> layout_lock(g_layout_mu);
  std::lock_guard<std::mutex> stage_lock(g_stage_mu);
  std::lock_guard<std::mutex> lock(g_mu);
  int cur = 0;
  cudaGetDevice(&cur);
  for (int dev = 0; dev < kMaxDevices; ++dev) {
    if (!g_ws[dev].ptr && !g_stage[dev].ptr && !g_layout[dev].ptr && !g_pad[dev].ptr &&
        !g_bwd[dev].ptr && g_tables[dev].empty())
      continue;
    cudaSetDevice(dev);
    if (g_ws[dev].ptr) cudaFree(g_ws[dev].ptr);
    if (g_stage[dev].ptr) cudaFree(g_stage[dev].ptr);
    if (g_layout[dev].ptr) cudaFree(g_layout[dev].ptr);
    if (g_pad[dev].ptr) cudaFree(g_pad[dev].ptr);
    if (g_bwd[dev].ptr) cudaFree(g_bwd[dev].ptr);
    for (PermTable& t : g_tables[dev]) cudaFree(t.dev_table);
    g_tables[dev].clear();
    g_ws[dev] = DevBuf();
    g_stage[dev] = DevBuf();
    g_layout[dev] = DevBuf();
    g_pad[dev] = DevBuf();
    g_bwd[dev] = DevBuf();
  }
  cudaSetDevice(cur);
}

int monarch_attn_check(cudaStream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return record_cuda(e);
  int dev;
  int st = current_device(&dev);
  if (st != MONARCH_OK) return st;
  int* p;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if ((st = status_word_locked(dev, &p)) != MONARCH_OK) return st;
  }
  int flag = 0;
  if ((e = cudaMemcpy(&flag, p, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return record_cuda(e);
  if (flag) {
    if ((e = cudaMemset(p, 0, sizeof(int))) != cudaSuccess) return record_cuda(e);
    return MONARCH_ERR_DEVICE_TIMEOUT;
  }
  return MONARCH_OK;
}

const char* monarch_attn_strerror(int status) {
  switch (status) {
    case MONARCH_OK: return "ok";
    case MONARCH_ERR_INVALID_ARG:
      return "invalid argument (null or misaligned pointer, overlapping output, or a size out "
             "of range)";
    case MONARCH_ERR_UNSUPPORTED: return "unsupported shape (d must be in [1, 256])";
    case MONARCH_ERR_CUDA: return t_err[0] ? t_err : "CUDA error";
    case MONARCH_ERR_DEVICE_TIMEOUT:
      return "a bounded device wait expired; the kernel stopped early and its output is invalid";
    case MONARCH_ERR_NO_MEMORY: return t_err[0] ? t_err : "workspace allocation failed";
    case MONARCH_ERR_SCRATCH_LIMIT:
      return "the shape needs more scratch than the 64 MiB static array of "
             "monarch_attn_fwd_noalloc holds";
    default: return "unknown status";
  }
}

int monarch_attn_last_launches(void) { return t_launches; }

int monarch_attn_selftest_timeout(unsigned long long limit_ns, cudaStream_t stream) {
  if (limit_ns > 10ull * 1000000000ull) return MONARCH_ERR_INVALID_ARG;
  int dev;
  int st = current_device(&dev);
  if (st != MONARCH_OK) return st;
  int* status;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if ((st = status_word_locked(dev, &status)) != MONARCH_OK) return st;
  }
  cudaError_t e = monarch::tc_selftest_timeout(status, limit_ns, stream);
  return e == cudaSuccess ? MONARCH_OK : record_cuda(e);
}

int monarch_attn_version(void) { return (0 << 16) | 2; }

}  // extern "C"
