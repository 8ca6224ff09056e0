// C ABI of libgdn.so: argument validation, dispatch to the kernels, the
// versioned state blob, device status, launch counting and the profiler.
//
// Every entry point validates all of its arguments on the host before it
// launches anything, so an error leaves every buffer untouched ("fail before
// unsafe or partial execution" and "without mutating session state":
// DS4Server issue #95, implementation comment).
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <cmath>
#include <mutex>
#include <string>
#include <tuple>
#include <vector>

#include "../../include/gdn.h"
#include "internal.h"

namespace {

thread_local std::string g_err;

gdn_status fail(gdn_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

gdn_status cuda_fail(cudaError_t e, const char* what) {
  return fail(GDN_E_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

std::atomic<int64_t> g_launches{0};

struct Profiler {
  std::mutex mu;
  bool on = false;
  std::vector<std::tuple<int, cudaEvent_t, cudaEvent_t>> pending;
  std::vector<cudaEvent_t> pool;
  int64_t count[GDN_K_COUNT] = {};
  double ms[GDN_K_COUNT] = {};
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }
  // resolve every pending pair (blocks until they have completed)
  void drain() {
    for (auto& p : pending) {
      float t = 0.f;
      cudaEventSynchronize(std::get<2>(p));
      if (cudaEventElapsedTime(&t, std::get<1>(p), std::get<2>(p)) == cudaSuccess) {
        count[std::get<0>(p)] += 1;
        ms[std::get<0>(p)] += t;
      }
      pool.push_back(std::get<1>(p));
      pool.push_back(std::get<2>(p));
    }
    pending.clear();
  }
};
Profiler g_prof;

struct EventPair {
  cudaEvent_t start, stop;
};

// Device-side words: the status word kernels set instead of trapping, and
// the checksum accumulator used to verify device-resident blobs.  Their
// device addresses are looked up once per device.
__device__ int32_t g_status_word;
__device__ unsigned long long g_checksum_word;

constexpr int kMaxDevices = 64;
int32_t* g_status_ptr[kMaxDevices];
unsigned long long* g_checksum_ptr[kMaxDevices];
int g_device_ok[kMaxDevices];  // 0 unknown, 1 ok, -1 unsupported
std::mutex g_dev_mu;

gdn_status check_device(int* dev_out = nullptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(GDN_E_DEVICE, "no usable CUDA device: %s", cudaGetErrorString(e));
  }
  if (dev < 0 || dev >= kMaxDevices) return fail(GDN_E_DEVICE, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (g_device_ok[dev] == 0) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0) {
      g_device_ok[dev] = -1;
    } else if (cudaGetSymbolAddress((void**)&g_status_ptr[dev], g_status_word) != cudaSuccess ||
               cudaGetSymbolAddress((void**)&g_checksum_ptr[dev], g_checksum_word) != cudaSuccess) {
      cudaGetLastError();
      return fail(GDN_E_CUDA, "cannot resolve device symbols on device %d", dev);
    } else {
      g_device_ok[dev] = 1;
    }
  }
  if (g_device_ok[dev] < 0) return fail(GDN_E_DEVICE, "device %d is not an sm_100 (B200) device", dev);
  if (dev_out) *dev_out = dev;
  return GDN_OK;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

gdn_status check_cfg(const gdn_config* cfg, gdn::Dims* d) {
  if (!cfg) return fail(GDN_E_INVAL, "cfg is NULL");
  if (cfg->num_k_heads <= 0 || cfg->num_v_heads <= 0 || cfg->head_k_dim <= 0 || cfg->head_v_dim <= 0 ||
      cfg->conv_width <= 0)
    return fail(GDN_E_INVAL, "geometry fields must be positive");
  if (cfg->num_v_heads % cfg->num_k_heads != 0)
    return fail(GDN_E_INVAL, "num_v_heads (%d) must be a multiple of num_k_heads (%d)", cfg->num_v_heads,
                cfg->num_k_heads);
  if (!(cfg->l2_eps >= 0.f) || !std::isfinite(cfg->l2_eps) || !(cfg->norm_eps >= 0.f) ||
      !std::isfinite(cfg->norm_eps) || !std::isfinite(cfg->q_scale))
    return fail(GDN_E_INVAL, "epsilons must be finite and >= 0, q_scale finite");
  if (cfg->io_dtype != GDN_F32 && cfg->io_dtype != GDN_BF16)
    return fail(GDN_E_UNSUPPORTED, "io_dtype %d is not GDN_F32 or GDN_BF16", cfg->io_dtype);
  if (cfg->conv_width != 4) return fail(GDN_E_UNSUPPORTED, "conv_width %d (only 4 is built)", cfg->conv_width);
  if (cfg->head_k_dim != cfg->head_v_dim ||
      (cfg->head_k_dim != 32 && cfg->head_k_dim != 64 && cfg->head_k_dim != 128))
    return fail(GDN_E_UNSUPPORTED, "head dims %d/%d (built: d_k == d_v in {32, 64, 128})", cfg->head_k_dim,
                cfg->head_v_dim);
  if ((int64_t)cfg->num_v_heads * cfg->head_v_dim > (1 << 24) || cfg->num_k_heads > (1 << 16))
    return fail(GDN_E_UNSUPPORTED, "head counts too large");
  d->Hk = cfg->num_k_heads;
  d->Hv = cfg->num_v_heads;
  d->dk = cfg->head_k_dim;
  d->dv = cfg->head_v_dim;
  d->W = cfg->conv_width;
  d->G = cfg->num_v_heads / cfg->num_k_heads;
  d->C = 2LL * d->Hk * d->dk + (int64_t)d->Hv * d->dv;
  d->l2_eps = cfg->l2_eps;
  d->norm_eps = cfg->norm_eps;
  d->q_scale = cfg->q_scale;
  return GDN_OK;
}

gdn_status check_ptr(const void* p, const char* name) {
  if (!p) return fail(GDN_E_INVAL, "%s is NULL", name);
  if (!aligned16(p)) return fail(GDN_E_INVAL, "%s is not 16-byte aligned", name);
  return GDN_OK;
}

// a and b are read one element at a time: natural alignment of the io dtype suffices.
gdn_status check_gate_ptr(const void* p, const char* name, const gdn_config* cfg) {
  if (!p) return fail(GDN_E_INVAL, "%s is NULL", name);
  const uintptr_t m = cfg->io_dtype == GDN_BF16 ? 1u : 3u;
  if ((uintptr_t)p & m) return fail(GDN_E_INVAL, "%s is not aligned to its element size", name);
  return GDN_OK;
}

gdn_status check_params(const gdn_params* prm) {
  if (!prm) return fail(GDN_E_INVAL, "params is NULL");
  gdn_status s;
  if ((s = check_ptr(prm->conv_w, "params.conv_w")) != GDN_OK) return s;
  if ((s = check_ptr(prm->A_log, "params.A_log")) != GDN_OK) return s;
  if ((s = check_ptr(prm->dt_bias, "params.dt_bias")) != GDN_OK) return s;
  if ((s = check_ptr(prm->norm_w, "params.norm_w")) != GDN_OK) return s;
  return GDN_OK;
}

constexpr int32_t kMaxSeqs = 65535;  // grid-dimension limit of the per-sequence conv launches

// cu_seqlens_host: cu[0] = 0, non-decreasing.  Returns total tokens, max length.
gdn_status check_cu(const int32_t* cu_dev, const int32_t* cu_host, int32_t N, int64_t* total, int32_t* max_len) {
  if (N <= 0 || N > kMaxSeqs) return fail(GDN_E_INVAL, "num_seqs %d outside 1..%d", N, kMaxSeqs);
  if (!cu_dev || !cu_host) return fail(GDN_E_INVAL, "cu_seqlens_dev and cu_seqlens_host are both required");
  if (((uintptr_t)cu_dev & 3u) != 0) return fail(GDN_E_INVAL, "cu_seqlens_dev is not 4-byte aligned");
  if (cu_host[0] != 0) return fail(GDN_E_INVAL, "cu_seqlens[0] = %d, expected 0", cu_host[0]);
  int32_t mx = 0;
  for (int32_t n = 0; n < N; ++n) {
    if (cu_host[n + 1] < cu_host[n])
      return fail(GDN_E_INVAL, "cu_seqlens decreases at %d (%d -> %d)", n, cu_host[n], cu_host[n + 1]);
    mx = std::max(mx, cu_host[n + 1] - cu_host[n]);
  }
  *total = cu_host[N];
  *max_len = mx;
  return GDN_OK;
}

int64_t chunk_bound(int64_t total_tokens, int32_t num_seqs, int32_t chunk_size) {
  return total_tokens / chunk_size + num_seqs + 1;
}

// Prefill paths (bf16, d = 128): the factored three-kernel path at chunk 64, the affine three-kernel
// path at chunk 16, 32 and 128 (and at 64 with GDN_PREFILL_AFFINE), one kernel per (sequence, value head)
// with GDN_PREFILL_FUSED (chunk 64); the token-recurrent kernel for everything else.
enum class Path { Wy, Split, Fused, Recurrent };

constexpr uint32_t kPathFlags = GDN_PREFILL_RECURRENT | GDN_PREFILL_FUSED | GDN_PREFILL_FACTORED | GDN_PREFILL_AFFINE;

Path prefill_path(const gdn::Dims& d, const gdn_config* cfg, int32_t chunk_size, uint32_t flags) {
  const bool bf16 = cfg->io_dtype == GDN_BF16;
  if (flags & GDN_PREFILL_RECURRENT) return Path::Recurrent;
  if (flags & GDN_PREFILL_FUSED)
    return gdn::prefill_chunked_supported(d, bf16, chunk_size) ? Path::Fused : Path::Recurrent;
  if (flags & GDN_PREFILL_AFFINE)
    return gdn::prefill_wy_supported(d, bf16, chunk_size) ? Path::Wy : Path::Recurrent;
  if (gdn::prefill_chunked_supported(d, bf16, chunk_size)) return Path::Split;  // chunk 64 (factored)
  if (gdn::prefill_wy_supported(d, bf16, chunk_size)) return Path::Wy;
  return Path::Recurrent;
}

// rows of the schedule's chunks: the affine path schedules tiles of 64 or 128 rows
int32_t sched_rows(Path p, int32_t chunk_size) { return p == Path::Wy ? gdn::wy_tile(chunk_size) : chunk_size; }

// schedule, then (three-kernel paths only) the intermediates of the chunked form
size_t prefill_ws_bytes(const gdn::Dims& d, Path p, int64_t total_tokens, int32_t num_seqs, int32_t chunk_size) {
  const int64_t chunks = chunk_bound(total_tokens, num_seqs, sched_rows(p, chunk_size));
  const size_t sched = gdn::schedule_layout(num_seqs, chunks).total_bytes;
  if (p == Path::Split) {  // one window of chunks at a time
    const int64_t w = gdn::split_window_chunks(chunks);
    return sched + gdn::split_layout(d, std::min<int64_t>(total_tokens, w * chunk_size), w).total_bytes;
  }
  if (p == Path::Wy) {  // one window of tiles at a time
    const int64_t w = gdn::wy_window_tiles(chunks, chunk_size);
    return sched + gdn::wy_layout(d, std::min<int64_t>(total_tokens, w * gdn::wy_tile(chunk_size)), w, chunk_size)
                       .total_bytes;
  }
  return sched;
}

// what gdn_prefill_workspace_size reports: enough for every path a flag can select
size_t prefill_ws_query(const gdn::Dims& d, const gdn_config* cfg, int64_t total_tokens, int32_t num_seqs,
                        int32_t chunk_size) {
  size_t m = 0;
  for (uint32_t f : {0u, (uint32_t)GDN_PREFILL_FACTORED, (uint32_t)GDN_PREFILL_AFFINE, (uint32_t)GDN_PREFILL_FUSED})
    m = std::max(m, prefill_ws_bytes(d, prefill_path(d, cfg, chunk_size, f), total_tokens, num_seqs, chunk_size));
  return m;
}

// ---------------------------------------------------------------- state blob
constexpr char kMagic[8] = {'G', 'D', 'N', 'S', 'T', 'A', 'T', 'E'};
constexpr uint32_t kBlobVersion = 1;
constexpr int32_t kLayoutId = 1;  // payload = conv history [W-1][C_conv] (io dtype) ++ state [Hv][d_v][d_k] (fp32)

struct BlobHeader {
  char magic[8];
  uint32_t version;
  uint32_t header_bytes;
  int32_t num_k_heads, num_v_heads, head_k_dim, head_v_dim, conv_width;
  int32_t io_dtype;
  int32_t state_dtype;  // 0 = fp32
  int32_t layout_id;
  uint64_t conv_bytes;
  uint64_t state_bytes;
  uint64_t checksum;
  uint8_t reserved[56];
};
static_assert(sizeof(BlobHeader) == 128, "blob header is 128 bytes");

size_t io_bytes(const gdn_config* cfg) { return cfg->io_dtype == GDN_BF16 ? 2 : 4; }
size_t conv_seq_bytes(const gdn::Dims& d, const gdn_config* cfg) { return (size_t)(d.W - 1) * d.C * io_bytes(cfg); }
size_t state_seq_bytes(const gdn::Dims& d) { return (size_t)d.Hv * d.dv * d.dk * sizeof(float); }

bool is_device_ptr(const void* p) {
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return attr.type == cudaMemoryTypeDevice || attr.type == cudaMemoryTypeManaged;
}

}  // namespace

// ------------------------------------------------------------------ LaunchScope
namespace gdn {
void set_error_message(const char* msg) { g_err = msg; }

size_t prefill_fused_ws_bytes(int64_t total_tokens, int32_t num_seqs, int32_t chunk_size) {
  return schedule_layout(num_seqs, chunk_bound(total_tokens, num_seqs, chunk_size)).total_bytes;
}

LaunchScope::LaunchScope(int kernel_id, cudaStream_t s) : id(kernel_id), stream(s), token(nullptr) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (g_prof.on) {
    std::lock_guard<std::mutex> lk(g_prof.mu);
    EventPair* ep = new EventPair{g_prof.get(), g_prof.get()};
    if (ep->start && ep->stop && cudaEventRecord(ep->start, s) == cudaSuccess) {
      token = ep;
    } else {
      if (ep->start) g_prof.pool.push_back(ep->start);
      if (ep->stop) g_prof.pool.push_back(ep->stop);
      delete ep;
    }
  }
}
LaunchScope::~LaunchScope() {
  if (token) {
    EventPair* ep = (EventPair*)token;
    std::lock_guard<std::mutex> lk(g_prof.mu);
    cudaEventRecord(ep->stop, stream);
    g_prof.pending.emplace_back(id, ep->start, ep->stop);
    delete ep;
  }
}
}  // namespace gdn

// ------------------------------------------------------------------ entry points
extern "C" {

int32_t gdn_abi_version(void) { return GDN_ABI_VERSION; }
const char* gdn_last_error(void) { return g_err.c_str(); }
int64_t gdn_launch_count(void) { return g_launches.load(); }
void gdn_launch_count_reset(void) { g_launches.store(0); }

const char* gdn_kernel_name(int32_t id) {
  static const char* names[GDN_K_COUNT] = {"conv_prefill",    "conv_step",       "conv_history", "schedule",
                                           "prefill_recurrent", "prefill_chunked", "decode",       "state_checksum",
                                           "split_conv",        "split_prep",      "split_chain",
                                           "slot_copy",         "gemm",            "seqpar",
                                           "diag",              "wy_conv",         "wy_prep",
                                           "wy_chain"};
  return (id >= 0 && id < GDN_K_COUNT) ? names[id] : "unknown";
}

gdn_status gdn_profiler_enable(int32_t enable) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  g_prof.on = enable != 0;
  return GDN_OK;
}

gdn_status gdn_profiler_reset(void) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  g_prof.drain();
  for (int i = 0; i < GDN_K_COUNT; ++i) {
    g_prof.count[i] = 0;
    g_prof.ms[i] = 0.0;
  }
  return GDN_OK;
}

gdn_status gdn_profiler_read(int32_t kernel_id, int64_t* launches, double* total_ms) {
  if (kernel_id < 0 || kernel_id >= GDN_K_COUNT || !launches || !total_ms)
    return fail(GDN_E_INVAL, "bad profiler query");
  std::lock_guard<std::mutex> lk(g_prof.mu);
  g_prof.drain();
  *launches = g_prof.count[kernel_id];
  *total_ms = g_prof.ms[kernel_id];
  return GDN_OK;
}

gdn_status gdn_get_device_status(int32_t* code, gdn_stream_t stream) {
  if (!code) return fail(GDN_E_INVAL, "code is NULL");
  int dev = 0;
  gdn_status s = check_device(&dev);
  if (s != GDN_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  int32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, g_status_ptr[dev], sizeof(v), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess && v != 0) e = cudaMemsetAsync(g_status_ptr[dev], 0, sizeof(int32_t), st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
  *code = v;
  return GDN_OK;
}

gdn_status gdn_debug_wait_expiry(uint32_t limit_us, gdn_stream_t stream) {
  if (limit_us < 1 || limit_us > 1000000u) return fail(GDN_E_INVAL, "limit_us %u outside 1..1000000", limit_us);
  int dev = 0;
  gdn_status s = check_device(&dev);
  if (s != GDN_OK) return s;
  cudaError_t e = gdn::launch_wait_expiry((uint64_t)limit_us * 1000ull, g_status_ptr[dev], (cudaStream_t)stream);
  return e == cudaSuccess ? GDN_OK : cuda_fail(e, "gdn_debug_wait_expiry launch");
}

gdn_status gdn_conv_prefill(const gdn_config* cfg, const void* x, const float* conv_w,
                            const int32_t* cu_seqlens_dev, const int32_t* cu_seqlens_host, int32_t num_seqs,
                            void* conv_state, void* y, gdn_stream_t stream) {
  gdn::Dims d;
  gdn_status s;
  if ((s = check_cfg(cfg, &d)) != GDN_OK) return s;
  int64_t total = 0;
  int32_t max_len = 0;
  if ((s = check_cu(cu_seqlens_dev, cu_seqlens_host, num_seqs, &total, &max_len)) != GDN_OK) return s;
  if ((s = check_ptr(conv_w, "conv_w")) != GDN_OK || (s = check_ptr(conv_state, "conv_state")) != GDN_OK) return s;
  if (total > 0 && ((s = check_ptr(x, "x")) != GDN_OK || (s = check_ptr(y, "y")) != GDN_OK)) return s;
  if ((s = check_device()) != GDN_OK) return s;
  const bool bf16 = cfg->io_dtype == GDN_BF16;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = gdn::launch_conv_prefill(d, bf16, x, conv_w, cu_seqlens_dev, num_seqs, max_len, conv_state, y, st);
  if (e == cudaSuccess) e = gdn::launch_conv_history(d, bf16, x, cu_seqlens_dev, num_seqs, false, conv_state, st);
  return e == cudaSuccess ? GDN_OK : cuda_fail(e, "gdn_conv_prefill launch");
}

gdn_status gdn_conv_step(const gdn_config* cfg, const void* x, const float* conv_w, int32_t num_seqs,
                         void* conv_state, void* y, gdn_stream_t stream) {
  gdn::Dims d;
  gdn_status s;
  if ((s = check_cfg(cfg, &d)) != GDN_OK) return s;
  if (num_seqs <= 0 || num_seqs > kMaxSeqs) return fail(GDN_E_INVAL, "num_seqs %d outside 1..%d", num_seqs, kMaxSeqs);
  if ((s = check_ptr(x, "x")) != GDN_OK || (s = check_ptr(conv_w, "conv_w")) != GDN_OK ||
      (s = check_ptr(conv_state, "conv_state")) != GDN_OK || (s = check_ptr(y, "y")) != GDN_OK)
    return s;
  if ((s = check_device()) != GDN_OK) return s;
  cudaError_t e = gdn::launch_conv_step(d, cfg->io_dtype == GDN_BF16, x, conv_w, num_seqs, conv_state, y,
                                        (cudaStream_t)stream);
  return e == cudaSuccess ? GDN_OK : cuda_fail(e, "gdn_conv_step launch");
}

gdn_status gdn_prefill_workspace_size(const gdn_config* cfg, int64_t total_tokens, int32_t num_seqs,
                                      int32_t chunk_size, size_t* bytes) {
  gdn::Dims d;
  gdn_status s;
  if ((s = check_cfg(cfg, &d)) != GDN_OK) return s;
  if (!bytes) return fail(GDN_E_INVAL, "bytes is NULL");
  if (total_tokens < 0 || num_seqs <= 0 || num_seqs > kMaxSeqs) return fail(GDN_E_INVAL, "bad sizes");
  if (chunk_size != 16 && chunk_size != 32 && chunk_size != 64 && chunk_size != 128)
    return fail(GDN_E_INVAL, "chunk_size %d (16, 32, 64 or 128)", chunk_size);
  *bytes = prefill_ws_query(d, cfg, total_tokens, num_seqs, chunk_size);
  return GDN_OK;
}

gdn_status gdn_prefill(const gdn_config* cfg, const gdn_params* params, const void* qkv, const void* z,
                       const void* a, const void* b, const int32_t* cu_seqlens_dev, const int32_t* cu_seqlens_host,
                       int32_t num_seqs, int32_t chunk_size, uint32_t flags, void* conv_state, float* state,
                       void* o, void* workspace, size_t workspace_bytes, gdn_stream_t stream) {
  gdn::Dims d;
  gdn_status s;
  if ((s = check_cfg(cfg, &d)) != GDN_OK) return s;
  if ((s = check_params(params)) != GDN_OK) return s;
  if (chunk_size != 16 && chunk_size != 32 && chunk_size != 64 && chunk_size != 128)
    return fail(GDN_E_INVAL, "chunk_size %d (16, 32, 64 or 128)", chunk_size);
  const uint32_t known = GDN_ZERO_INIT_STATE | GDN_ZERO_INIT_CONV | kPathFlags;
  if (flags & ~known) return fail(GDN_E_INVAL, "unknown flags 0x%x", flags & ~known);
  if (__builtin_popcount(flags & kPathFlags) > 1)
    return fail(GDN_E_INVAL, "flags 0x%x select more than one prefill path", flags & kPathFlags);
  int64_t total = 0;
  int32_t max_len = 0;
  if ((s = check_cu(cu_seqlens_dev, cu_seqlens_host, num_seqs, &total, &max_len)) != GDN_OK) return s;
  if ((s = check_ptr(conv_state, "conv_state")) != GDN_OK || (s = check_ptr(state, "state")) != GDN_OK) return s;
  if (total > 0) {
    if ((s = check_ptr(qkv, "qkv")) != GDN_OK || (s = check_ptr(z, "z")) != GDN_OK ||
        (s = check_gate_ptr(a, "a", cfg)) != GDN_OK || (s = check_gate_ptr(b, "b", cfg)) != GDN_OK ||
        (s = check_ptr(o, "o")) != GDN_OK)
      return s;
  }
  const Path path = prefill_path(d, cfg, chunk_size, flags);
  const bool split = path == Path::Split || path == Path::Wy;
  const size_t need = prefill_ws_bytes(d, path, total, num_seqs, chunk_size);
  if (workspace_bytes < need || (need > 0 && !workspace))
    return fail(GDN_E_WORKSPACE, "workspace of %zu bytes at %p, need %zu", workspace_bytes, workspace, need);
  if (((uintptr_t)workspace & 255u) != 0) return fail(GDN_E_WORKSPACE, "workspace is not 256-byte aligned");
  int dev = 0;
  if ((s = check_device(&dev)) != GDN_OK) return s;
  if (total == 0) return GDN_OK;  // every sequence empty: nothing changes

  cudaStream_t st = (cudaStream_t)stream;
  const bool bf16 = cfg->io_dtype == GDN_BF16;
  const bool zero_state = flags & GDN_ZERO_INIT_STATE, zero_conv = flags & GDN_ZERO_INIT_CONV;
  const int32_t rows = sched_rows(path, chunk_size);  // rows per scheduled chunk (tiles on the affine path)
  int64_t chunks = 0;
  for (int32_t n = 0; n < num_seqs; ++n) chunks += (cu_seqlens_host[n + 1] - cu_seqlens_host[n] + rows - 1) / rows;
  const gdn::ScheduleLayout L = gdn::schedule_layout(num_seqs, chunks);
  cudaError_t e = cudaSuccess;
  const int32_t* order = nullptr;
  if (num_seqs > 1) {  // one sequence needs neither an order nor a chunk map
    e = gdn::launch_schedule(cu_seqlens_dev, num_seqs, rows, chunks, workspace, st);
    order = (const int32_t*)((const char*)workspace + L.order_off);
  }
  const bool chunked = path == Path::Fused;
  // intermediates start after the schedule sized for the chunk bound (the layout the size query assumed)
  const size_t sched = gdn::schedule_layout(num_seqs, chunk_bound(total, num_seqs, rows)).total_bytes;
  if (e == cudaSuccess && path == Path::Wy) {
    e = gdn::launch_prefill_wy(d, chunk_size, params->conv_w, params->A_log, params->dt_bias, params->norm_w, qkv,
                               z, a, b, cu_seqlens_dev, cu_seqlens_host, order,
                               num_seqs > 1 ? (const int32_t*)((const char*)workspace + L.chunk_off_off) : nullptr,
                               num_seqs > 1 ? (const int4*)((const char*)workspace + L.chunk_map_off) : nullptr,
                               num_seqs, total, chunks, zero_state, zero_conv, conv_state, state, o,
                               (char*)workspace + sched, g_status_ptr[dev], st);
  } else if (e == cudaSuccess && path == Path::Split) {
    e = gdn::launch_prefill_split(d, params->conv_w, params->A_log, params->dt_bias, params->norm_w, qkv, z, a, b,
                                  cu_seqlens_dev, cu_seqlens_host, order,
                                  num_seqs > 1 ? (const int32_t*)((const char*)workspace + L.chunk_off_off) : nullptr,
                                  num_seqs > 1 ? (const int4*)((const char*)workspace + L.chunk_map_off) : nullptr,
                                  num_seqs, total, chunks,
                                  zero_state, zero_conv, conv_state, state, o, (char*)workspace + sched,
                                  g_status_ptr[dev], st);
  } else if (e == cudaSuccess && chunked)
    e = gdn::launch_prefill_chunked(d, params->conv_w, params->A_log, params->dt_bias, params->norm_w, qkv, z, a, b,
                                    cu_seqlens_dev, order, num_seqs, total, zero_state, zero_conv, conv_state, state,
                                    o, g_status_ptr[dev], st);
  else if (e == cudaSuccess)
    e = gdn::launch_prefill_recurrent(d, bf16, params->conv_w, params->A_log, params->dt_bias, params->norm_w, qkv,
                                      z, a, b, cu_seqlens_dev, order, num_seqs, zero_state, zero_conv, conv_state,
                                      state, o, st);
  // The three-kernel path writes each non-empty sequence's new history in its prep kernel; an empty
  // sequence keeps its history unless the history is to start from zeros.
  bool empty_zeroed = false;
  for (int32_t n = 0; n < num_seqs && zero_conv; ++n) empty_zeroed |= cu_seqlens_host[n + 1] == cu_seqlens_host[n];
  if (e == cudaSuccess && (!split || empty_zeroed))
    e = gdn::launch_conv_history(d, bf16, qkv, cu_seqlens_dev, num_seqs, zero_conv, conv_state, st);
  return e == cudaSuccess ? GDN_OK : cuda_fail(e, "gdn_prefill launch");
}

namespace {

gdn_status check_slots(const int32_t* slots_dev, int32_t num_slots, int32_t num_seqs) {
  if (!slots_dev) return fail(GDN_E_INVAL, "state_indices is NULL");
  if ((uintptr_t)slots_dev & 3u) return fail(GDN_E_INVAL, "state_indices is not 4-byte aligned");
  if (num_slots <= 0 || num_slots > kMaxSeqs) return fail(GDN_E_INVAL, "num_slots %d out of range", num_slots);
  (void)num_seqs;
  return GDN_OK;
}

gdn_status decode_step_impl(const gdn_config* cfg, const gdn_params* params, const void* qkv, const void* z,
                            const void* a, const void* b, int32_t num_seqs, gdn::Slots slots, void* conv_state,
                            float* state, void* o, gdn_stream_t stream, const char* what) {
  gdn::Dims d;
  gdn_status s;
  if ((s = check_cfg(cfg, &d)) != GDN_OK) return s;
  if ((s = check_params(params)) != GDN_OK) return s;
  if (num_seqs <= 0 || (int64_t)num_seqs * d.Hk > 0x7fffffffLL)
    return fail(GDN_E_INVAL, "num_seqs %d out of range", num_seqs);
  if ((s = check_ptr(qkv, "qkv")) != GDN_OK || (s = check_ptr(z, "z")) != GDN_OK ||
      (s = check_gate_ptr(a, "a", cfg)) != GDN_OK || (s = check_gate_ptr(b, "b", cfg)) != GDN_OK ||
      (s = check_ptr(conv_state, "conv_state")) != GDN_OK || (s = check_ptr(state, "state")) != GDN_OK ||
      (s = check_ptr(o, "o")) != GDN_OK)
    return s;
  int dev = 0;
  if ((s = check_device(&dev)) != GDN_OK) return s;
  cudaError_t e = gdn::launch_decode_step(d, cfg->io_dtype == GDN_BF16, params->conv_w, params->A_log,
                                          params->dt_bias, params->norm_w, qkv, z, a, b, num_seqs, slots, conv_state,
                                          state, o, g_status_ptr[dev], (cudaStream_t)stream);
  return e == cudaSuccess ? GDN_OK : cuda_fail(e, what);
}

gdn_status decode_multi_impl(const gdn_config* cfg, const gdn_params* params, const void* qkv, const void* z,
                             const void* a, const void* b, int32_t num_seqs, int32_t num_tokens, int32_t commit,
                             const int32_t* accept_dev, gdn::Slots slots, void* conv_state, float* state, void* o,
                             gdn_stream_t stream, const char* what) {
  gdn::Dims d;
  gdn_status s;
  if ((s = check_cfg(cfg, &d)) != GDN_OK) return s;
  if ((s = check_params(params)) != GDN_OK) return s;
  if (num_seqs <= 0 || (int64_t)num_seqs * d.Hk > 0x7fffffffLL)
    return fail(GDN_E_INVAL, "num_seqs %d out of range", num_seqs);
  if (num_tokens < 1 || num_tokens > GDN_MAX_DRAFT_TOKENS)
    return fail(GDN_E_INVAL, "num_tokens %d outside [1, %d]", num_tokens, GDN_MAX_DRAFT_TOKENS);
  if (!commit && accept_dev) return fail(GDN_E_INVAL, "accept must be NULL when commit == 0");
  if (d.dk != 128 || d.dv != 128)
    return fail(GDN_E_UNSUPPORTED, "gdn_decode_multi runs d_k = d_v = 128 only (got %d, %d)", d.dk, d.dv);
  if ((s = check_ptr(qkv, "qkv")) != GDN_OK || (s = check_ptr(z, "z")) != GDN_OK ||
      (s = check_gate_ptr(a, "a", cfg)) != GDN_OK || (s = check_gate_ptr(b, "b", cfg)) != GDN_OK ||
      (s = check_ptr(conv_state, "conv_state")) != GDN_OK || (s = check_ptr(state, "state")) != GDN_OK ||
      (s = check_ptr(o, "o")) != GDN_OK)
    return s;
  if (accept_dev && ((uintptr_t)accept_dev & 3u)) return fail(GDN_E_INVAL, "accept is not 4-byte aligned");
  int dev = 0;
  if ((s = check_device(&dev)) != GDN_OK) return s;
  cudaError_t e = gdn::launch_decode_multi(d, cfg->io_dtype == GDN_BF16, params->conv_w, params->A_log,
                                           params->dt_bias, params->norm_w, qkv, z, a, b, num_seqs, num_tokens,
                                           accept_dev, commit ? 1 : 0, slots, conv_state, state, o, g_status_ptr[dev],
                                           (cudaStream_t)stream);
  return e == cudaSuccess ? GDN_OK : cuda_fail(e, what);
}

}  // namespace

gdn_status gdn_decode_step(const gdn_config* cfg, const gdn_params* params, const void* qkv, const void* z,
                           const void* a, const void* b, int32_t num_seqs, void* conv_state, float* state, void* o,
                           gdn_stream_t stream) {
  return decode_step_impl(cfg, params, qkv, z, a, b, num_seqs, gdn::Slots{nullptr, 0}, conv_state, state, o, stream,
                          "gdn_decode_step launch");
}

gdn_status gdn_decode_step_indexed(const gdn_config* cfg, const gdn_params* params, const void* qkv, const void* z,
                                   const void* a, const void* b, int32_t num_seqs, const int32_t* state_indices,
                                   int32_t num_slots, void* conv_state, float* state, void* o, gdn_stream_t stream) {
  gdn_status s;
  if ((s = check_slots(state_indices, num_slots, num_seqs)) != GDN_OK) return s;
  return decode_step_impl(cfg, params, qkv, z, a, b, num_seqs, gdn::Slots{state_indices, num_slots}, conv_state,
                          state, o, stream, "gdn_decode_step_indexed launch");
}

gdn_status gdn_decode_multi(const gdn_config* cfg, const gdn_params* params, const void* qkv, const void* z,
                            const void* a, const void* b, int32_t num_seqs, int32_t num_tokens, int32_t commit,
                            const int32_t* accept_dev, void* conv_state, float* state, void* o,
                            gdn_stream_t stream) {
  return decode_multi_impl(cfg, params, qkv, z, a, b, num_seqs, num_tokens, commit, accept_dev,
                           gdn::Slots{nullptr, 0}, conv_state, state, o, stream, "gdn_decode_multi launch");
}

gdn_status gdn_decode_multi_indexed(const gdn_config* cfg, const gdn_params* params, const void* qkv, const void* z,
                                    const void* a, const void* b, int32_t num_seqs, int32_t num_tokens,
                                    int32_t commit, const int32_t* accept_dev, const int32_t* state_indices,
                                    int32_t num_slots, void* conv_state, float* state, void* o,
                                    gdn_stream_t stream) {
  gdn_status s;
  if ((s = check_slots(state_indices, num_slots, num_seqs)) != GDN_OK) return s;
  return decode_multi_impl(cfg, params, qkv, z, a, b, num_seqs, num_tokens, commit, accept_dev,
                           gdn::Slots{state_indices, num_slots}, conv_state, state, o, stream,
                           "gdn_decode_multi_indexed launch");
}

namespace {

// workspace of an indexed prefill: gdn_prefill's, then the batch's state and conv-history buffers
struct IndexedLayout {
  size_t state_off, conv_off, total;
};
IndexedLayout indexed_layout(const gdn::Dims& d, bool bf16, size_t base, int32_t num_seqs) {
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  IndexedLayout L;
  L.state_off = al(base);
  L.conv_off = al(L.state_off + (size_t)num_seqs * d.Hv * d.dv * d.dk * sizeof(float));
  L.total = al(L.conv_off + (size_t)num_seqs * (d.W - 1) * d.C * (bf16 ? 2 : 4));
  return L;
}

}  // namespace

gdn_status gdn_prefill_indexed_workspace_size(const gdn_config* cfg, int64_t total_tokens, int32_t num_seqs,
                                              int32_t chunk_size, size_t* bytes) {
  size_t base = 0;
  gdn_status s = gdn_prefill_workspace_size(cfg, total_tokens, num_seqs, chunk_size, &base);
  if (s != GDN_OK) return s;
  gdn::Dims d;
  if ((s = check_cfg(cfg, &d)) != GDN_OK) return s;
  *bytes = indexed_layout(d, cfg->io_dtype == GDN_BF16, base, num_seqs).total;
  return GDN_OK;
}

gdn_status gdn_prefill_indexed(const gdn_config* cfg, const gdn_params* params, const void* qkv, const void* z,
                               const void* a, const void* b, const int32_t* cu_seqlens_dev,
                               const int32_t* cu_seqlens_host, int32_t num_seqs, const int32_t* state_indices,
                               int32_t num_slots, int32_t chunk_size, uint32_t flags, void* conv_state, float* state,
                               void* o, void* workspace, size_t workspace_bytes, gdn_stream_t stream) {
  // every check gdn_prefill makes comes first, so that an error launches nothing
  gdn::Dims d;
  gdn_status s;
  if ((s = check_cfg(cfg, &d)) != GDN_OK) return s;
  if ((s = check_params(params)) != GDN_OK) return s;
  if ((s = check_slots(state_indices, num_slots, num_seqs)) != GDN_OK) return s;
  if (chunk_size != 16 && chunk_size != 32 && chunk_size != 64 && chunk_size != 128)
    return fail(GDN_E_INVAL, "chunk_size %d (16, 32, 64 or 128)", chunk_size);
  const uint32_t known = GDN_ZERO_INIT_STATE | GDN_ZERO_INIT_CONV | kPathFlags;
  if (flags & ~known) return fail(GDN_E_INVAL, "unknown flags 0x%x", flags & ~known);
  if (__builtin_popcount(flags & kPathFlags) > 1)
    return fail(GDN_E_INVAL, "flags 0x%x select more than one prefill path", flags & kPathFlags);
  int64_t total = 0;
  int32_t max_len = 0;
  if ((s = check_cu(cu_seqlens_dev, cu_seqlens_host, num_seqs, &total, &max_len)) != GDN_OK) return s;
  if ((s = check_ptr(conv_state, "conv_state")) != GDN_OK || (s = check_ptr(state, "state")) != GDN_OK) return s;
  if (total > 0) {
    if ((s = check_ptr(qkv, "qkv")) != GDN_OK || (s = check_ptr(z, "z")) != GDN_OK ||
        (s = check_gate_ptr(a, "a", cfg)) != GDN_OK || (s = check_gate_ptr(b, "b", cfg)) != GDN_OK ||
        (s = check_ptr(o, "o")) != GDN_OK)
      return s;
  }
  const bool bf16 = cfg->io_dtype == GDN_BF16;
  const size_t base = prefill_ws_bytes(d, prefill_path(d, cfg, chunk_size, flags), total, num_seqs, chunk_size);
  const IndexedLayout L = indexed_layout(d, bf16, base, num_seqs);
  if (workspace_bytes < L.total || !workspace)
    return fail(GDN_E_WORKSPACE, "workspace of %zu bytes at %p, need %zu", workspace_bytes, workspace, L.total);
  if (((uintptr_t)workspace & 255u) != 0) return fail(GDN_E_WORKSPACE, "workspace is not 256-byte aligned");
  int dev = 0;
  if ((s = check_device(&dev)) != GDN_OK) return s;
  if (total == 0) return GDN_OK;  // every sequence empty: nothing changes

  cudaStream_t st = (cudaStream_t)stream;
  const gdn::Slots slots{state_indices, num_slots};
  float* buf_state = (float*)((char*)workspace + L.state_off);
  void* buf_conv = (char*)workspace + L.conv_off;
  cudaError_t e = gdn::launch_slot_copy(d, bf16, slots, num_seqs, true, state, conv_state, buf_state, buf_conv,
                                        g_status_ptr[dev], st);
  if (e != cudaSuccess) return cuda_fail(e, "gdn_prefill_indexed gather");
  if ((s = gdn_prefill(cfg, params, qkv, z, a, b, cu_seqlens_dev, cu_seqlens_host, num_seqs, chunk_size, flags,
                       buf_conv, buf_state, o, workspace, L.state_off, stream)) != GDN_OK)
    return s;
  e = gdn::launch_slot_copy(d, bf16, slots, num_seqs, false, state, conv_state, buf_state, buf_conv,
                            g_status_ptr[dev], st);
  return e == cudaSuccess ? GDN_OK : cuda_fail(e, "gdn_prefill_indexed scatter");
}

namespace {

int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      n <= 0) {
    cudaGetLastError();
    n = 148;
  }
  return n;
}

gdn_status seqpar_check(const gdn_config* cfg, gdn::Dims* d, int64_t total_tokens, int32_t segments) {
  gdn_status s;
  if ((s = check_cfg(cfg, d)) != GDN_OK) return s;
  if (cfg->io_dtype != GDN_BF16 || d->dk != 128 || d->dv != 128)
    return fail(GDN_E_UNSUPPORTED, "the sequence-parallel prefill runs bf16 io with d_k = d_v = 128");
  if (total_tokens < 0 || total_tokens > 0x7fffffffLL)
    return fail(GDN_E_INVAL, "total_tokens %lld out of range", (long long)total_tokens);
  if (segments < 0 || segments > 4096) return fail(GDN_E_INVAL, "segments %d outside 0..4096", segments);
  return GDN_OK;
}

}  // namespace

gdn_status gdn_prefill_seqpar_workspace_size(const gdn_config* cfg, int64_t total_tokens, int32_t segments,
                                             size_t* bytes) {
  gdn::Dims d;
  gdn_status s;
  if ((s = seqpar_check(cfg, &d, total_tokens, segments)) != GDN_OK) return s;
  if (!bytes) return fail(GDN_E_INVAL, "bytes is NULL");
  const int P = gdn::seqpar_segments(d, total_tokens, segments, device_sms());
  *bytes = gdn::seqpar_layout(d, total_tokens, P).total_bytes;
  return GDN_OK;
}

gdn_status gdn_prefill_seqpar(const gdn_config* cfg, const gdn_params* params, const void* qkv, const void* z,
                              const void* a, const void* b, int64_t total_tokens, int32_t segments, uint32_t flags,
                              void* conv_state, float* state, void* o, void* workspace, size_t workspace_bytes,
                              int32_t* segments_used, gdn_stream_t stream) {
  gdn::Dims d;
  gdn_status s;
  if ((s = seqpar_check(cfg, &d, total_tokens, segments)) != GDN_OK) return s;
  if ((s = check_params(params)) != GDN_OK) return s;
  const uint32_t known = GDN_ZERO_INIT_STATE | GDN_ZERO_INIT_CONV;
  if (flags & ~known) return fail(GDN_E_INVAL, "flags 0x%x: only GDN_ZERO_INIT_STATE and GDN_ZERO_INIT_CONV", flags);
  if ((s = check_ptr(conv_state, "conv_state")) != GDN_OK || (s = check_ptr(state, "state")) != GDN_OK) return s;
  if (total_tokens > 0) {
    if ((s = check_ptr(qkv, "qkv")) != GDN_OK || (s = check_ptr(z, "z")) != GDN_OK ||
        (s = check_gate_ptr(a, "a", cfg)) != GDN_OK || (s = check_gate_ptr(b, "b", cfg)) != GDN_OK ||
        (s = check_ptr(o, "o")) != GDN_OK)
      return s;
  }
  const int P = gdn::seqpar_segments(d, total_tokens, segments, device_sms());
  const size_t need = gdn::seqpar_layout(d, total_tokens, P).total_bytes;
  if (workspace_bytes < need || !workspace)
    return fail(GDN_E_WORKSPACE, "workspace of %zu bytes at %p, need %zu", workspace_bytes, workspace, need);
  if (((uintptr_t)workspace & 255u) != 0) return fail(GDN_E_WORKSPACE, "workspace is not 256-byte aligned");
  int dev = 0;
  if ((s = check_device(&dev)) != GDN_OK) return s;
  if (segments_used) *segments_used = P;
  if (total_tokens == 0) return GDN_OK;
  cudaError_t e = gdn::launch_prefill_seqpar(d, params->conv_w, params->A_log, params->dt_bias, params->norm_w, qkv,
                                             z, a, b, total_tokens, P, flags & GDN_ZERO_INIT_STATE,
                                             flags & GDN_ZERO_INIT_CONV, conv_state, state, o, workspace,
                                             g_status_ptr[dev], (cudaStream_t)stream);
  return e == cudaSuccess ? GDN_OK : cuda_fail(e, "gdn_prefill_seqpar launch");
}

}  // extern "C"

namespace {

// output k of a GEMM: columns [start, start + width) to ptr (row pitch ld elements)
void gemm_route(gdn::GemmOutputs& g, void* ptr, int64_t ld, int32_t width) {
  const int k = g.count++;
  g.ptr[k] = ptr;
  g.ld[k] = ld;
  g.start[k + 1] = g.start[k] + width;
  g.vec[k] = aligned16(ptr) && ld % 8 == 0 && g.start[k] % 8 == 0;
}

gdn_status gemm_impl(const void* x, int32_t M, int32_t K, const void* w, int32_t N, int32_t tile_n,
                     const gdn::GemmOutputs& out, gdn_stream_t stream, const char* what) {
  gdn_status s;
  if (M < 0 || N < 0) return fail(GDN_E_INVAL, "%s: M = %d, N = %d (must be >= 0)", what, M, N);
  if (K <= 0 || K % 8 != 0) return fail(GDN_E_INVAL, "%s: K = %d must be a positive multiple of 8", what, K);
  if (tile_n != 0 && (tile_n % 32 != 0 || tile_n < 32 || tile_n > 256))
    return fail(GDN_E_INVAL, "%s: tile_n %d (0, or a multiple of 32 up to 256)", what, tile_n);
  if ((s = check_ptr(x, "x")) != GDN_OK || (s = check_ptr(w, "w")) != GDN_OK) return s;
  for (int k = 0; k < out.count; ++k)
    if (!out.ptr[k] || ((uintptr_t)out.ptr[k] & 1u)) return fail(GDN_E_INVAL, "%s: output %d is NULL or odd", what, k);
  int dev = 0;
  if ((s = check_device(&dev)) != GDN_OK) return s;
  if (M == 0 || N == 0) return GDN_OK;
  cudaError_t e = gdn::launch_gemm_bf16(x, M, K, w, N, tile_n, out, g_status_ptr[dev], (cudaStream_t)stream);
  return e == cudaSuccess ? GDN_OK : cuda_fail(e, what);
}

}  // namespace

extern "C" {

gdn_status gdn_gemm_bf16(const void* x, int32_t M, int32_t K, const void* w, int32_t N, void* y, int32_t tile_n,
                         gdn_stream_t stream) {
  gdn::GemmOutputs g{};
  gemm_route(g, y, N, N);
  return gemm_impl(x, M, K, w, N, tile_n, g, stream, "gdn_gemm_bf16");
}

gdn_status gdn_project_in(const gdn_config* cfg, const void* x, int32_t num_tokens, int32_t hidden,
                          const void* w_in, void* qkv, void* z, void* a, void* b, gdn_stream_t stream) {
  gdn::Dims d;
  gdn_status s;
  if ((s = check_cfg(cfg, &d)) != GDN_OK) return s;
  if (cfg->io_dtype != GDN_BF16) return fail(GDN_E_UNSUPPORTED, "gdn_project_in runs bf16 io only");
  const int64_t hvd = (int64_t)d.Hv * d.dv, n = d.C + hvd + 2LL * d.Hv;
  if (n > 0x7fffffffLL) return fail(GDN_E_UNSUPPORTED, "projection width %lld too large", (long long)n);
  if ((s = check_ptr(qkv, "qkv")) != GDN_OK || (s = check_ptr(z, "z")) != GDN_OK ||
      (s = check_gate_ptr(a, "a", cfg)) != GDN_OK || (s = check_gate_ptr(b, "b", cfg)) != GDN_OK)
    return s;
  gdn::GemmOutputs g{};
  gemm_route(g, qkv, d.C, (int32_t)d.C);
  gemm_route(g, z, hvd, (int32_t)hvd);
  gemm_route(g, a, d.Hv, d.Hv);
  gemm_route(g, b, d.Hv, d.Hv);
  return gemm_impl(x, num_tokens, hidden, w_in, (int32_t)n, 0, g, stream, "gdn_project_in");
}

gdn_status gdn_project_out(const gdn_config* cfg, const void* o, int32_t num_tokens, const void* w_out,
                           int32_t hidden, void* y, gdn_stream_t stream) {
  gdn::Dims d;
  gdn_status s;
  if ((s = check_cfg(cfg, &d)) != GDN_OK) return s;
  if (cfg->io_dtype != GDN_BF16) return fail(GDN_E_UNSUPPORTED, "gdn_project_out runs bf16 io only");
  const int64_t hvd = (int64_t)d.Hv * d.dv;
  if (hvd > 0x7fffffffLL) return fail(GDN_E_UNSUPPORTED, "Hv * d_v too large");
  if ((s = check_ptr(y, "y")) != GDN_OK) return s;
  gdn::GemmOutputs g{};
  gemm_route(g, y, hidden, hidden);
  return gemm_impl(o, num_tokens, (int32_t)hvd, w_out, hidden, 0, g, stream, "gdn_project_out");
}

gdn_status gdn_state_blob_size(const gdn_config* cfg, size_t* bytes) {
  gdn::Dims d;
  gdn_status s;
  if ((s = check_cfg(cfg, &d)) != GDN_OK) return s;
  if (!bytes) return fail(GDN_E_INVAL, "bytes is NULL");
  *bytes = sizeof(BlobHeader) + conv_seq_bytes(d, cfg) + state_seq_bytes(d);
  return GDN_OK;
}

gdn_status gdn_state_save(const gdn_config* cfg, const void* conv_state, const float* state, int32_t seq,
                          void* blob, size_t blob_bytes, gdn_stream_t stream) {
  gdn::Dims d;
  gdn_status s;
  if ((s = check_cfg(cfg, &d)) != GDN_OK) return s;
  if (seq < 0) return fail(GDN_E_INVAL, "seq %d < 0", seq);
  if ((s = check_ptr(conv_state, "conv_state")) != GDN_OK || (s = check_ptr(state, "state")) != GDN_OK) return s;
  if (!blob) return fail(GDN_E_INVAL, "blob is NULL");
  const size_t cb = conv_seq_bytes(d, cfg), sb = state_seq_bytes(d);
  if (blob_bytes < sizeof(BlobHeader) + cb + sb)
    return fail(GDN_E_INVAL, "blob of %zu bytes, need %zu", blob_bytes, sizeof(BlobHeader) + cb + sb);
  if ((s = check_device()) != GDN_OK) return s;
  BlobHeader hdr;
  memset(&hdr, 0, sizeof(hdr));
  memcpy(hdr.magic, kMagic, 8);
  hdr.version = kBlobVersion;
  hdr.header_bytes = sizeof(BlobHeader);
  hdr.num_k_heads = d.Hk;
  hdr.num_v_heads = d.Hv;
  hdr.head_k_dim = d.dk;
  hdr.head_v_dim = d.dv;
  hdr.conv_width = d.W;
  hdr.io_dtype = cfg->io_dtype;
  hdr.state_dtype = 0;
  hdr.layout_id = kLayoutId;
  hdr.conv_bytes = cb;
  hdr.state_bytes = sb;
  const char* conv_src = (const char*)conv_state + (size_t)seq * cb;
  const char* state_src = (const char*)state + (size_t)seq * sb;
  char* payload = (char*)blob + sizeof(BlobHeader);
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  if (is_device_ptr(blob)) {
    e = cudaMemcpyAsync(blob, &hdr, sizeof(hdr), cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaMemcpyAsync(payload, conv_src, cb, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess) e = cudaMemcpyAsync(payload + cb, state_src, sb, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess)
      e = gdn::launch_checksum(payload, cb + sb, (unsigned long long*)((char*)blob + offsetof(BlobHeader, checksum)),
                               st);
  } else {
    e = cudaMemcpyAsync(payload, conv_src, cb, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaMemcpyAsync(payload + cb, state_src, sb, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess) {
      hdr.checksum = gdn::host_checksum(payload, cb + sb);
      memcpy(blob, &hdr, sizeof(hdr));
    }
  }
  return e == cudaSuccess ? GDN_OK : cuda_fail(e, "gdn_state_save");
}

gdn_status gdn_state_restore(const gdn_config* cfg, const void* blob, size_t blob_bytes, int32_t seq,
                             void* conv_state, float* state, gdn_stream_t stream) {
  gdn::Dims d;
  gdn_status s;
  if ((s = check_cfg(cfg, &d)) != GDN_OK) return s;
  if (seq < 0) return fail(GDN_E_INVAL, "seq %d < 0", seq);
  if ((s = check_ptr(conv_state, "conv_state")) != GDN_OK || (s = check_ptr(state, "state")) != GDN_OK) return s;
  if (!blob) return fail(GDN_E_INVAL, "blob is NULL");
  if (blob_bytes < sizeof(BlobHeader)) return fail(GDN_E_BLOB_FORMAT, "blob of %zu bytes has no header", blob_bytes);
  const bool dev_blob = is_device_ptr(blob);
  cudaStream_t st = (cudaStream_t)stream;
  BlobHeader hdr;
  if (dev_blob) {
    cudaError_t e = cudaMemcpyAsync(&hdr, blob, sizeof(hdr), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "reading the blob header");
  } else {
    memcpy(&hdr, blob, sizeof(hdr));
  }
  if (memcmp(hdr.magic, kMagic, 8) != 0) return fail(GDN_E_BLOB_FORMAT, "bad blob magic");
  if (hdr.version != kBlobVersion) return fail(GDN_E_BLOB_VERSION, "blob format version %u, expected %u", hdr.version, kBlobVersion);
  if (hdr.header_bytes != sizeof(BlobHeader) || hdr.layout_id != kLayoutId)
    return fail(GDN_E_BLOB_FORMAT, "blob header size %u / layout id %d not recognised", hdr.header_bytes, hdr.layout_id);
  if (hdr.num_k_heads != d.Hk || hdr.num_v_heads != d.Hv || hdr.head_k_dim != d.dk || hdr.head_v_dim != d.dv ||
      hdr.conv_width != d.W || hdr.io_dtype != cfg->io_dtype || hdr.state_dtype != 0)
    return fail(GDN_E_BLOB_GEOMETRY,
                "blob saved for Hk=%d Hv=%d dk=%d dv=%d W=%d io=%d state=%d, config has Hk=%d Hv=%d dk=%d dv=%d W=%d io=%d",
                hdr.num_k_heads, hdr.num_v_heads, hdr.head_k_dim, hdr.head_v_dim, hdr.conv_width, hdr.io_dtype,
                hdr.state_dtype, d.Hk, d.Hv, d.dk, d.dv, d.W, cfg->io_dtype);
  const size_t cb = conv_seq_bytes(d, cfg), sb = state_seq_bytes(d);
  if (hdr.conv_bytes != cb || hdr.state_bytes != sb || blob_bytes < sizeof(BlobHeader) + cb + sb)
    return fail(GDN_E_BLOB_FORMAT, "blob payload sizes do not match the geometry");
  const char* payload = (const char*)blob + sizeof(BlobHeader);
  uint64_t sum = 0;
  int dev = 0;
  if (dev_blob) {
    if ((s = check_device(&dev)) != GDN_OK) return s;
    unsigned long long v = 0;
    cudaError_t e = cudaMemsetAsync(g_checksum_ptr[dev], 0, sizeof(v), st);
    if (e == cudaSuccess) e = gdn::launch_checksum(payload, cb + sb, g_checksum_ptr[dev], st);
    if (e == cudaSuccess) e = cudaMemcpyAsync(&v, g_checksum_ptr[dev], sizeof(v), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "checksumming the device blob");
    sum = v;
  } else {
    sum = gdn::host_checksum(payload, cb + sb);
  }
  if (sum != hdr.checksum) return fail(GDN_E_BLOB_CHECKSUM, "blob checksum mismatch");
  if ((s = check_device()) != GDN_OK) return s;
  const cudaMemcpyKind kind = dev_blob ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
  cudaError_t e = cudaMemcpyAsync((char*)conv_state + (size_t)seq * cb, payload, cb, kind, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync((char*)state + (size_t)seq * sb, payload + cb, sb, kind, st);
  return e == cudaSuccess ? GDN_OK : cuda_fail(e, "gdn_state_restore copy");
}

}  // extern "C"
