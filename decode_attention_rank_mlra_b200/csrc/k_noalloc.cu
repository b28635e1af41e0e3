// mlra_decode_attn_noalloc: split-KV attention plus combine with the scratch
// held in a fixed device array owned by this library, for callers that cannot
// allocate device memory themselves.
//
// Who needs it: code that runs where cudaMalloc is not available to it -- a
// plugin inside a host framework that owns all device memory through its own
// allocator, or a serving process that reserves every free byte of HBM for the
// KV cache at start-up and must not allocate afterwards (cudaMalloc may also
// synchronise the device, which a latency-bound decode loop cannot afford).
//
// The scratch array below (16 MiB) is created when the library is loaded and
// held by every GPU that loads it until the process exits.
#include "mlra_internal.cuh"

#include <mutex>

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;

// Device-side scratch shared by every call of mlra_decode_attn_noalloc.  In
// host code this name is only a stand-in: its device address comes from
// cudaGetSymbolAddress (once per device and context, below).
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDev = 64;
std::mutex g_mu;
struct ScratchAddr {
  void* ctx;  // the context the address was looked up in
  void* ptr;
};
ScratchAddr g_scratch[kMaxDev] = {};

// The current context (CUcontext) through the driver entry point, or NULL.
void* current_context() {
  using GetCurrent = int (*)(void**);
  static GetCurrent fn = nullptr;
  static bool looked = false;
  if (!looked) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<GetCurrent>(p);
    looked = true;
  }
  void* ctx = nullptr;
  if (!fn || fn(&ctx) != 0) return nullptr;
  return ctx;
}

// Device address of the scratch on the current device.  Looked up with that
// device current on the first call, and again whenever the device's context
// has changed since (a cudaDeviceReset destroys the context and the module
// that holds the array; the next context loads it again, possibly elsewhere).
mlra_status_t scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return MLRA_ERR_NO_DEVICE;
  // (no context may be current yet in this thread: then it is looked up, which
  // also makes the device's primary context current)
  void* ctx = current_context();
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch[dev].ptr || ctx == nullptr || g_scratch[dev].ctx != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return MLRA_ERR_CUDA;
    g_scratch[dev] = ScratchAddr{current_context(), p};
  }
  *out = g_scratch[dev].ptr;
  return MLRA_OK;
}

__global__ void copy_status_kernel(const int32_t* __restrict__ src, int32_t* __restrict__ dst) {
  *dst = *src;
}

}  // namespace

extern "C" mlra_status_t mlra_decode_attn_noalloc(
    const mlra_config_t* cfg, const float* q_abs, const void* q_rope, const void* kv_cache,
    int64_t num_pages, const int32_t* page_table, int32_t max_pages, const int32_t* seqlens,
    int32_t batch, float* o_latent, float* lse, int32_t* device_status, mlra_stream_t stream) {
  size_t need = 0;
  mlra_status_t st = mlra_workspace_size(cfg, batch, &need);
  if (st != MLRA_OK) return st;
  if (need > kNoAllocScratchBytes) return MLRA_ERR_WORKSPACE;  // batch too large for the array
  void* scratch = nullptr;
  st = scratch_for_current_device(&scratch);
  if (st != MLRA_OK) return st;
  // The plan kernel launched by mlra_decode_attn rewrites the header (and
  // clears the error word) before anything reads the array, and every split
  // partial the combine reads is written by the attention kernel first, so
  // nothing left from a previous call is ever consumed.
  st = mlra_decode_attn(cfg, q_abs, q_rope, kv_cache, num_pages, page_table, max_pages, seqlens,
                        batch, scratch, kNoAllocScratchBytes, stream);
  if (st != MLRA_OK) return st;
  st = mlra_splitkv_combine(cfg, scratch, kNoAllocScratchBytes, batch, o_latent, lse, stream);
  if (st != MLRA_OK) return st;
  if (device_status) {
    copy_status_kernel<<<1, 1, 0, (cudaStream_t)stream>>>(static_cast<const int32_t*>(scratch),
                                                          device_status);
    if (cudaGetLastError() != cudaSuccess) return MLRA_ERR_CUDA;
  }
  return MLRA_OK;
}
