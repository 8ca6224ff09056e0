// gdn_prefill_noalloc: gdn_prefill without a caller-provided workspace.
//
// Some callers cannot hand this library any scratch device memory: a host
// runtime whose device memory is entirely owned by another allocator (a
// framework's caching allocator or a serving engine's pre-reserved pool) that
// offers no way to borrow from it, or latency-critical code that must not call
// cudaMalloc/cudaFree because those calls can synchronise the whole device.
// For them the prefill's scratch lives in a fixed array in this library's own
// device memory, reserved when the library is loaded onto a GPU and held by
// every GPU that loads it until the process exits.  Nothing is allocated at
// call time.
#include <cstdio>
#include <mutex>

#include "../../include/gdn.h"
#include "internal.h"

namespace {

constexpr size_t kScratchBytes = GDN_NOALLOC_SCRATCH_BYTES;

// The scratch array.  In host code this name is only a host-side stand-in for
// the symbol, not a device address; the device address comes from
// cudaGetSymbolAddress below and is what the kernels receive.
static __device__ __align__(256) unsigned char g_prefill_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device, looked up once
// per device with that device current.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_prefill_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" GDN_API gdn_status gdn_prefill_noalloc(const gdn_config* cfg, const gdn_params* params, const void* qkv,
                                                  const void* z, const void* a, const void* b,
                                                  const int32_t* cu_seqlens_dev, const int32_t* cu_seqlens_host,
                                                  int32_t num_seqs, int32_t chunk_size, uint32_t flags,
                                                  void* conv_state, float* state, void* o, gdn_stream_t stream) {
  // gdn_prefill_workspace_size validates cfg, num_seqs and chunk_size; the
  // remaining arguments are validated by gdn_prefill before anything runs.
  size_t need = 0;
  gdn_status s = gdn_prefill_workspace_size(cfg, 0, num_seqs, chunk_size, &need);
  if (s != GDN_OK) return s;
  if (!cu_seqlens_host) {
    gdn::set_error_message("gdn_prefill_noalloc: cu_seqlens_host is NULL");
    return GDN_E_INVAL;
  }
  // the entry point runs the single-kernel path; another path flag would need a workspace of its own
  const uint32_t other_paths = flags & (GDN_PREFILL_RECURRENT | GDN_PREFILL_FACTORED | GDN_PREFILL_AFFINE);
  if (other_paths) {
    char msg[192];
    snprintf(msg, sizeof(msg),
             "gdn_prefill_noalloc: flags 0x%x select another prefill path; this entry point runs the "
             "single-kernel path (GDN_PREFILL_FUSED) only",
             other_paths);
    gdn::set_error_message(msg);
    return GDN_E_INVAL;
  }
  // cu_seqlens_host must be valid before its last entry sizes the schedule
  if (cu_seqlens_host[0] != 0) {
    gdn::set_error_message("gdn_prefill_noalloc: cu_seqlens_host[0] is not 0");
    return GDN_E_INVAL;
  }
  for (int32_t n = 0; n < num_seqs; ++n) {
    if (cu_seqlens_host[n + 1] < cu_seqlens_host[n]) {
      gdn::set_error_message("gdn_prefill_noalloc: cu_seqlens_host decreases");
      return GDN_E_INVAL;
    }
  }
  // the single-kernel chunked path needs only the schedule as scratch
  need = gdn::prefill_fused_ws_bytes(cu_seqlens_host[num_seqs], num_seqs, chunk_size);
  if (need > kScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "gdn_prefill_noalloc: this problem needs %zu bytes of scratch but the built-in scratch array holds %zu "
             "(GDN_NOALLOC_SCRATCH_BYTES); use gdn_prefill with a workspace",
             need, kScratchBytes);
    gdn::set_error_message(msg);
    return GDN_E_WORKSPACE;
  }
  void* ws = nullptr;
  cudaError_t e = scratch_address(&ws);
  if (e != cudaSuccess) {
    cudaGetLastError();
    char msg[256];
    snprintf(msg, sizeof(msg), "gdn_prefill_noalloc: cannot resolve the scratch array on this device: %s",
             cudaGetErrorString(e));
    gdn::set_error_message(msg);
    return GDN_E_DEVICE;
  }
  return gdn_prefill(cfg, params, qkv, z, a, b, cu_seqlens_dev, cu_seqlens_host, num_seqs, chunk_size,
                     flags | GDN_PREFILL_FUSED, conv_state, state, o, ws, kScratchBytes, stream);
}
