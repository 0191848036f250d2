// vt_attention_static: the stand-alone attention entry point for callers that cannot
// allocate device memory.  Some callers cannot call cudaMalloc or hand the library a
// workspace: code that runs inside a host framework whose allocator owns all device
// memory, or a plugin interface that passes only its input and output buffers.  This
// entry point keeps its scratch (the rotated q and k and the transposed v) in a
// file-scope device array instead, and allocates nothing.
//
// The array is part of the library image, so every GPU that loads libvt holds its
// kStaticScratchBytes until the process exits.  Every call uses the same array and
// leaves its own contents behind; nothing in it has to start at zero, because each
// call writes every byte it later reads.  Calls whose GPU work overlaps (two streams,
// or two threads on one device) race on the array and must be serialised by the
// caller.
#include <mutex>

#include "internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB

// Host code must not take this name as a device address: on the host it names a
// stand-in object.  The device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

inline size_t round_up256(size_t x) { return (x + 255) & ~size_t(255); }

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device, looked up once per
// device (the first call on each device does this set-up).
vt_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    vt::set_error_message("vt_attention_static: cudaGetDevice failed");
    return VT_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    vt::set_error_message("vt_attention_static: device index out of range");
    return VT_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || !p) {
      vt::set_error_message("vt_attention_static: cudaGetSymbolAddress of the static scratch failed");
      return VT_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return VT_OK;
}

}  // namespace

extern "C" {

vt_status vt_attention_static_max_bytes(size_t* out) {
  if (!out) {
    vt::set_error_message("vt_attention_static_max_bytes: out is NULL");
    return VT_ERR_INVALID_ARG;
  }
  *out = kStaticScratchBytes;
  return VT_OK;
}

vt_status vt_attention_static(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int D,
                              const int32_t* pos_thw, const int32_t* sections, float theta, float scale,
                              void* stream) {
  vt_status s = vt::check_attention_dims(B, H, N, D, scale);
  if (s != VT_OK) return s;
  if (!q || !k || !v || !o) {
    vt::set_error_message("vt_attention_static: NULL operand");
    return VT_ERR_INVALID_ARG;
  }
  if (((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v) |
        reinterpret_cast<uintptr_t>(o)) & 15u) != 0) {
    vt::set_error_message("vt_attention_static: device pointers must be 16-byte aligned");
    return VT_ERR_INVALID_ARG;
  }
  int sec[3] = {0, 0, 0};
  if (pos_thw) {
    if (!sections) {
      vt::set_error_message("vt_attention_static: sections must be given with pos_thw");
      return VT_ERR_INVALID_ARG;
    }
    for (int a = 0; a < 3; ++a) {
      sec[a] = sections[a];
      if (sec[a] < 0 || (sec[a] & 1)) {
        vt::set_error_message("vt_attention_static: rope sections must be even");
        return VT_ERR_INVALID_ARG;
      }
    }
    if (sec[0] + sec[1] + sec[2] != D || !(theta > 0.f)) {
      vt::set_error_message("vt_attention_static: sections must sum to head_dim and theta be positive");
      return VT_ERR_INVALID_ARG;
    }
  }
  // B * H * N < 2^31 (checked above) keeps these products far inside 64 bits.
  const int ldv = (N + 7) & ~7;
  const size_t part = round_up256(static_cast<size_t>(B) * H * D * ldv * 2);
  if (part > kStaticScratchBytes / 3) {
    vt::set_error_message("vt_attention_static: problem needs more scratch than the 32 MiB static array "
                          "(3 * B*H*D*ceil8(N) * 2 bytes); use vt_attention with a workspace");
    return VT_ERR_WORKSPACE;
  }
  void* base = nullptr;
  if ((s = scratch_address(&base)) != VT_OK) return s;
  char* w = static_cast<char*>(base);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = vt::run_attention_prep(q, k, v, w, w + part, w + 2 * part, B, H, N, D, ldv, pos_thw, sec, theta, st)))
    return s;
  vt::AttnParams a{w, w + part, w + 2 * part, o, B, H, N, D, ldv, scale};
  return vt::run_attention(a, st);
}

}  // extern "C"
