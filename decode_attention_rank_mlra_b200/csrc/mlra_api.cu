// Host side of the C ABI declared in include/mlra.h: argument validation,
// workspace layout, kernel selection and launches.  No allocation, no host
// synchronisation (except mlra_get_device_error).
#include "dispatch.h"

#include <stdlib.h>
#include <string.h>

#include <mutex>

using namespace mlra;

namespace {

constexpr int kMaxDevices = 64;

int num_sms_current(int* dev_out) {
  static int cache[kMaxDevices] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  if (dev_out) *dev_out = dev;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    cache[dev] = n;
  }
  return cache[dev];
}

bool device_is_sm100(int dev) {
  static int cache[kMaxDevices] = {0};  // 0 unknown, 1 yes, 2 no
  if (dev < 0 || dev >= kMaxDevices) return false;
  if (cache[dev] == 0) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cache[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return cache[dev] == 1;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

mlra_status_t check_cfg(const mlra_config_t* c) {
  if (!c) return MLRA_ERR_INVALID_ARG;
  if (c->n_blocks < 1 || c->d_cb < 1 || c->d_r < 0 || c->n_heads < 1 || c->d_h < 1)
    return MLRA_ERR_INVALID_ARG;
  if (c->dtype != MLRA_F32 && c->dtype != MLRA_BF16) return MLRA_ERR_INVALID_ARG;
  if (!(c->softmax_scale == c->softmax_scale) || !(c->branch_scale == c->branch_scale))
    return MLRA_ERR_INVALID_ARG;  // NaN
  if (c->d_h > 128 || (c->d_h % 8) != 0 || (c->d_cb % 8) != 0) return MLRA_ERR_UNSUPPORTED;
  return MLRA_OK;
}

// 1 = tensor core, 2 = SIMT, 0 = unsupported.  The fp32 cache and the bf16
// shapes the tensor-core kernels do not take (head counts other than 16, 32,
// 64 or multiples of 128; latent blocks other than 128, or 512 for one block)
// run on the fp32 SIMT kernel.
int choose_kernel(const mlra_config_t& c, int dev) {
  if (c.dtype == MLRA_BF16 && device_is_sm100(dev) && tc_supported(c)) return 1;
  if (simt_supported(c)) return 2;
  return 0;
}

// Tensor-core absorption / output projection on this device for this config?
// (bf16 with d_h = 128; the SIMT kernels take the rest.)
bool use_proj_tc(const mlra_config_t& c) {
  if (!proj_tc_supported(c)) return false;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  return device_is_sm100(dev);
}

// MLRA_TEST_STALL_TILE=<k>: tests of the failure path only (see
// DecodeArgs::stall_tile).  Read once per process.
int test_stall_tile() {
  static int v = -2;
  if (v == -2) {
    const char* e = getenv("MLRA_TEST_STALL_TILE");
    v = e ? atoi(e) : -1;
    if (v < 0) v = -1;
  }
  return v;
}

struct Grid { int kind, n_groups, ctas_per_group; };

mlra_status_t plan_grid(const mlra_config_t& c, Grid* g) {
  int dev = 0;
  const int sms = num_sms_current(&dev);
  if (sms <= 0) return MLRA_ERR_NO_DEVICE;
  g->kind = choose_kernel(c, dev);
  if (g->kind == 1) tc_grid(c, sms, &g->n_groups, &g->ctas_per_group);
  else if (g->kind == 2) simt_grid(c, sms, &g->n_groups, &g->ctas_per_group);
  else return MLRA_ERR_UNSUPPORTED;
  return MLRA_OK;
}

WsLayout layout_for(const mlra_config_t& c, int batch, const Grid& g) {
  return ws_layout(batch, c.n_heads, c.n_blocks, c.d_cb, batch + g.ctas_per_group);
}

mlra_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? MLRA_OK : MLRA_ERR_CUDA; }

// q_abs = alpha * W_uk q_nope on the tensor cores where they apply, else SIMT.
mlra_status_t absorb(const mlra_config_t& c, const void* q_nope, const void* w_uk, float* q_abs,
                     int batch, float alpha, cudaStream_t s) {
  if (use_proj_tc(c) && aligned(q_nope, 16)) {
    cudaError_t e = launch_absorb_tc(c, q_nope, w_uk, q_abs, batch, alpha, s);
    if (e != cudaErrorNotSupported) return from_cuda(e);
  }
  return from_cuda(launch_absorb(c, q_nope, w_uk, q_abs, batch, alpha, s));
}

// Device address of the host range [p, p + bytes) when it is page-locked and
// mapped into the current device's address space (checked at both ends), else
// NULL, in which case no kernel ever dereferences it.
const void* mapped_host_range(const void* p, size_t bytes) {
  if (!p || bytes == 0) return nullptr;
  cudaPointerAttributes a0{}, a1{};
  const char* last = static_cast<const char*>(p) + (bytes - 1);
  if (cudaPointerGetAttributes(&a0, p) != cudaSuccess ||
      cudaPointerGetAttributes(&a1, last) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  if (a0.type != cudaMemoryTypeHost || a1.type != cudaMemoryTypeHost || !a0.devicePointer ||
      !a1.devicePointer)
    return nullptr;
  if (static_cast<const char*>(a1.devicePointer) - static_cast<const char*>(a0.devicePointer) !=
      ptrdiff_t(bytes - 1))
    return nullptr;
  return a0.devicePointer;
}

// mlra_decode_step's workspace: the decode workspace, then its own buffers,
// each starting on a 256-byte boundary.
struct StepLayout {
  size_t attn, q_abs, o_lat, q_nope, q_rope, seqlens, out, total;
};

StepLayout step_layout(const mlra_config_t& c, int batch, const Grid& g) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t esz = c.dtype == MLRA_BF16 ? 2 : 4;
  const size_t bh = size_t(batch) * c.n_heads, K = size_t(c.n_blocks) * c.d_cb;
  StepLayout s;
  s.attn = up(layout_for(c, batch, g).total);
  s.q_abs = s.attn;
  s.o_lat = s.q_abs + up(bh * K * 4);
  s.q_nope = s.o_lat + up(bh * K * 4);
  s.q_rope = s.q_nope + up(bh * c.d_h * esz);
  s.seqlens = s.q_rope + up(bh * c.d_r * esz);
  s.out = s.seqlens + up(size_t(batch) * 4);
  s.total = s.out + up(bh * c.d_h * 4);
  return s;
}


// ---------------------------------------------------------------------------
// mlra_decode_step: one call's arguments, the transfers its host buffers need,
// and the launches, replayed as a CUDA graph from the second call with the
// same arguments on.
struct StepCall {
  mlra_config_t cfg;
  const void *q_nope, *q_rope;
  const int32_t* seqlens;
  int32_t batch;
  const void *w_uk, *w_uv, *kv_cache;
  int64_t num_pages;
  const int32_t* page_table;
  int32_t max_pages;
  float* out;
  int32_t host_io;
  void* workspace;
  size_t workspace_bytes;
  StepLayout S;
  // resolved by resolve_step
  const void *k_q_nope, *k_q_rope;  // what the kernels read
  const int32_t* k_seqlens;
  StageCopy staged[3];
  int n_staged;
  StageCopy copies_in[3];  // pageable inputs: copy-engine transfers
  int n_copies_in;
  float* dev_out;
  bool copy_out;
};

// Host buffers: ranges the device can read in place (page-locked, mapped) move
// in one staging launch, others by copy-engine transfers; the output is
// written by the projection kernel straight into mapped host memory, else into
// the workspace and copied back.
void resolve_step(StepCall* c) {
  char* ws = static_cast<char*>(c->workspace);
  const size_t esz = c->cfg.dtype == MLRA_BF16 ? 2 : 4;
  const size_t bh = size_t(c->batch) * c->cfg.n_heads;
  c->k_q_nope = c->q_nope;
  c->k_q_rope = c->q_rope;
  c->k_seqlens = c->seqlens;
  c->n_staged = c->n_copies_in = 0;
  c->dev_out = c->out;
  c->copy_out = false;
  if (!c->host_io) return;
  const void* src[3] = {c->q_nope, c->q_rope, c->seqlens};
  const size_t off[3] = {c->S.q_nope, c->S.q_rope, c->S.seqlens};
  const size_t len[3] = {bh * c->cfg.d_h * esz, bh * c->cfg.d_r * esz, size_t(c->batch) * 4};
  for (int k = 0; k < 3; ++k) {
    if (const void* d = mapped_host_range(src[k], len[k]))
      c->staged[c->n_staged++] = StageCopy{d, ws + off[k], len[k]};
    else
      c->copies_in[c->n_copies_in++] = StageCopy{src[k], ws + off[k], len[k]};
  }
  c->k_q_nope = ws + c->S.q_nope;
  c->k_q_rope = ws + c->S.q_rope;
  c->k_seqlens = reinterpret_cast<const int32_t*>(ws + c->S.seqlens);
  if (void* d = const_cast<void*>(mapped_host_range(c->out, bh * c->cfg.d_h * 4))) {
    c->dev_out = static_cast<float*>(d);
  } else {
    c->dev_out = reinterpret_cast<float*>(ws + c->S.out);
    c->copy_out = true;
  }
}

mlra_status_t enqueue_step(const StepCall& c, cudaStream_t s) {
  char* ws = static_cast<char*>(c.workspace);
  mlra_stream_t stream = (mlra_stream_t)s;
  for (int k = 0; k < c.n_copies_in; ++k)
    if (cudaMemcpyAsync(c.copies_in[k].dst, c.copies_in[k].src, c.copies_in[k].bytes,
                        cudaMemcpyHostToDevice, s) != cudaSuccess)
      return MLRA_ERR_CUDA;
  if (c.n_staged > 0 && launch_stage(c.staged, c.n_staged, s) != cudaSuccess) return MLRA_ERR_CUDA;
  float* q_abs = reinterpret_cast<float*>(ws + c.S.q_abs);
  mlra_status_t st = mlra_absorb_q(&c.cfg, c.k_q_nope, c.w_uk, q_abs, c.batch, stream);
  if (st != MLRA_OK) return st;
  st = mlra_decode_attn(&c.cfg, q_abs, c.k_q_rope, c.kv_cache, c.num_pages, c.page_table,
                        c.max_pages, c.k_seqlens, c.batch, c.workspace, c.S.attn, stream);
  if (st != MLRA_OK) return st;
  // The fused kernel needs no latent output; where it does not apply, the
  // two-kernel fallback writes it to the workspace.
  st = mlra_combine_out_proj(&c.cfg, c.workspace, c.S.attn, c.batch, c.w_uv, c.dev_out, nullptr,
                             nullptr, stream);
  if (st == MLRA_ERR_UNSUPPORTED)
    st = mlra_combine_out_proj(&c.cfg, c.workspace, c.S.attn, c.batch, c.w_uv, c.dev_out,
                               reinterpret_cast<float*>(ws + c.S.o_lat), nullptr, stream);
  if (st != MLRA_OK || !c.copy_out) return st;
  const size_t bytes = size_t(c.batch) * c.cfg.n_heads * c.cfg.d_h * 4;
  return from_cuda(cudaMemcpyAsync(c.out, c.dev_out, bytes, cudaMemcpyDeviceToHost, s));
}

// The graph cache: a call whose transfers are all kernels (device buffers, or
// mapped host buffers) is keyed by everything it passes to the kernels.  The
// first call with a key runs its launches directly (which also sets the
// kernels' attributes), the second records them on a private stream and
// instantiates the graph, later ones replay it: one launch instead of five.
// The graph reads the lengths, queries and cache at replay time, so their
// contents may change between calls; their addresses may not.  A stream that
// the caller is capturing is never recorded into.  The cache holds a fixed
// number of graphs and never evicts one (a replay may still be running).
struct StepKey {
  mlra_config_t cfg;
  const void* p[10];
  int64_t num_pages;
  int32_t batch, max_pages, host_io, dev;
  size_t workspace_bytes;
};

bool same_key(const StepKey& a, const StepKey& b) {
  if (memcmp(&a.cfg, &b.cfg, sizeof(a.cfg)) != 0) return false;
  for (int i = 0; i < 10; ++i)
    if (a.p[i] != b.p[i]) return false;
  return a.num_pages == b.num_pages && a.batch == b.batch && a.max_pages == b.max_pages &&
         a.host_io == b.host_io && a.dev == b.dev && a.workspace_bytes == b.workspace_bytes;
}

struct StepGraph {
  StepKey key;
  int state;  // 1: seen once, 2: graph ready, -1: recording failed (run directly)
  cudaGraphExec_t exec;
};
constexpr int kStepGraphs = 64;
std::mutex g_step_mu;
StepGraph g_step_graphs[kStepGraphs];
int g_step_n = 0;
cudaStream_t g_capture_stream[kMaxDevices] = {};

mlra_status_t run_step(const StepCall& c, cudaStream_t s) {
  const bool graphable = c.n_copies_in == 0 && !c.copy_out;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (!graphable || cudaStreamIsCapturing(s, &cs) != cudaSuccess ||
      cs != cudaStreamCaptureStatusNone) {
    (void)cudaGetLastError();
    return enqueue_step(c, s);
  }
  StepKey k;
  memset(&k, 0, sizeof(k));
  k.cfg = c.cfg;
  const void* ps[10] = {c.q_nope, c.q_rope, c.seqlens, c.w_uk, c.w_uv, c.kv_cache,
                        c.page_table, c.out, c.workspace, c.dev_out};
  for (int i = 0; i < 10; ++i) k.p[i] = ps[i];
  k.num_pages = c.num_pages;
  k.batch = c.batch;
  k.max_pages = c.max_pages;
  k.host_io = c.host_io;
  k.workspace_bytes = c.workspace_bytes;
  if (cudaGetDevice(&k.dev) != cudaSuccess || k.dev < 0 || k.dev >= kMaxDevices)
    return enqueue_step(c, s);
  StepGraph* e = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_step_mu);
    for (int i = 0; i < g_step_n; ++i)
      if (same_key(g_step_graphs[i].key, k)) e = &g_step_graphs[i];
    if (e && e->state == 2) {
      const cudaGraphExec_t exec = e->exec;
      return from_cuda(cudaGraphLaunch(exec, s));
    }
    if (!e) {
      if (g_step_n < kStepGraphs) {
        g_step_graphs[g_step_n] = StepGraph{k, 1, nullptr};
        ++g_step_n;
      }
      return enqueue_step(c, s);
    }
    if (e->state != 1) return enqueue_step(c, s);
    // second call with this key: record it (under the lock, so that one thread
    // records and the others wait for the graph)
    cudaStream_t& cap = g_capture_stream[k.dev];
    bool ok = cap != nullptr ||
              cudaStreamCreateWithFlags(&cap, cudaStreamNonBlocking) == cudaSuccess;
    cudaGraph_t graph = nullptr;
    cudaGraphExec_t exec = nullptr;
    if (ok) ok = cudaStreamBeginCapture(cap, cudaStreamCaptureModeThreadLocal) == cudaSuccess;
    if (ok) {
      const mlra_status_t rec = enqueue_step(c, cap);
      const bool ended = cudaStreamEndCapture(cap, &graph) == cudaSuccess;
      ok = rec == MLRA_OK && ended && graph != nullptr &&
           cudaGraphInstantiate(&exec, graph, 0) == cudaSuccess;
    }
    if (graph) cudaGraphDestroy(graph);
    (void)cudaGetLastError();
    if (!ok) {
      if (exec) cudaGraphExecDestroy(exec);
      e->state = -1;
      return enqueue_step(c, s);
    }
    e->exec = exec;
    e->state = 2;
    return from_cuda(cudaGraphLaunch(exec, s));
  }
}

}  // namespace

extern "C" {

const char* mlra_status_string(mlra_status_t s) {
  switch (s) {
    case MLRA_OK: return "ok";
    case MLRA_ERR_INVALID_ARG: return "invalid argument";
    case MLRA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case MLRA_ERR_ALIGNMENT: return "pointer under-aligned";
    case MLRA_ERR_WORKSPACE: return "workspace too small or misaligned";
    case MLRA_ERR_CUDA: return "CUDA error";
    case MLRA_ERR_BAD_PAGE: return "page id out of range (device)";
    case MLRA_ERR_TIMEOUT: return "bounded wait expired (device)";
    case MLRA_ERR_NO_DEVICE: return "no usable CUDA device";
    case MLRA_ERR_RANGE: return "cache value outside the fp16 range of the tensor-core path (device)";
  }
  return "unknown status";
}

int32_t mlra_version(void) { return 10000; }

int32_t mlra_decode_kernel_kind(const mlra_config_t* cfg) {
  if (check_cfg(cfg) != MLRA_OK) return 0;
  Grid g;
  if (plan_grid(*cfg, &g) != MLRA_OK) return 0;
  return g.kind;
}

mlra_status_t mlra_absorb_q(const mlra_config_t* cfg, const void* q_nope, const void* w_uk,
                            float* q_abs, int32_t batch, mlra_stream_t stream) {
  mlra_status_t st = check_cfg(cfg);
  if (st != MLRA_OK) return st;
  if (batch < 0) return MLRA_ERR_INVALID_ARG;
  if (batch == 0) return MLRA_OK;
  if (!q_nope || !w_uk || !q_abs) return MLRA_ERR_INVALID_ARG;
  if (!aligned(w_uk, 16) || !aligned(q_nope, cfg->dtype == MLRA_BF16 ? 2 : 4) || !aligned(q_abs, 4))
    return MLRA_ERR_ALIGNMENT;
  return absorb(*cfg, q_nope, w_uk, q_abs, batch, 1.0f, (cudaStream_t)stream);
}

mlra_status_t mlra_absorb_q_rope(const mlra_config_t* cfg, const void* q_nope, const void* q_rope,
                                 const int32_t* positions, float alpha_q, float rope_theta,
                                 const void* w_uk, float* q_abs, void* q_rope_out, int32_t batch,
                                 mlra_stream_t stream) {
  mlra_status_t st = check_cfg(cfg);
  if (st != MLRA_OK) return st;
  if (batch < 0) return MLRA_ERR_INVALID_ARG;
  if (batch == 0) return MLRA_OK;
  if (!q_nope || !q_rope || !positions || !w_uk || !q_abs || !q_rope_out)
    return MLRA_ERR_INVALID_ARG;
  if (!(alpha_q == alpha_q) || !(rope_theta > 0.f) || cfg->d_r % 2 != 0 || cfg->d_r > 512)
    return MLRA_ERR_INVALID_ARG;
  const uintptr_t el = cfg->dtype == MLRA_BF16 ? 2 : 4;
  if (!aligned(w_uk, 16) || !aligned(q_nope, el) || !aligned(q_rope, el) ||
      !aligned(q_rope_out, el) || !aligned(q_abs, 4) || !aligned(positions, 4))
    return MLRA_ERR_ALIGNMENT;
  const size_t rope_bytes = size_t(batch) * cfg->n_heads * cfg->d_r * el;
  const char* a = static_cast<const char*>(q_rope);
  const char* b = static_cast<const char*>(q_rope_out);
  if (a != b && a < b + rope_bytes && b < a + rope_bytes) return MLRA_ERR_INVALID_ARG;  // overlap
  cudaStream_t s = (cudaStream_t)stream;
  st = absorb(*cfg, q_nope, w_uk, q_abs, batch, alpha_q, s);
  if (st != MLRA_OK) return st;
  return from_cuda(launch_query_rope(*cfg, q_rope, positions, alpha_q, double(rope_theta),
                                     q_rope_out, batch, s));
}

mlra_status_t mlra_workspace_size(const mlra_config_t* cfg, int32_t batch, size_t* bytes) {
  mlra_status_t st = check_cfg(cfg);
  if (st != MLRA_OK) return st;
  if (batch < 0 || !bytes) return MLRA_ERR_INVALID_ARG;
  Grid g;
  st = plan_grid(*cfg, &g);
  if (st != MLRA_OK) return st;
  *bytes = layout_for(*cfg, batch, g).total;
  return MLRA_OK;
}

mlra_status_t mlra_decode_attn(const mlra_config_t* cfg, const float* q_abs, const void* q_rope,
                               const void* kv_cache, int64_t num_pages,
                               const int32_t* page_table, int32_t max_pages,
                               const int32_t* seqlens, int32_t batch, void* workspace,
                               size_t workspace_bytes, mlra_stream_t stream) {
  mlra_status_t st = check_cfg(cfg);
  if (st != MLRA_OK) return st;
  if (batch < 0) return MLRA_ERR_INVALID_ARG;
  if (!workspace) return MLRA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MLRA_ERR_WORKSPACE;
  if (batch > 0 && (!q_abs || !q_rope || !kv_cache || !seqlens)) return MLRA_ERR_INVALID_ARG;
  if (max_pages < 1) return MLRA_ERR_INVALID_ARG;
  if (page_table) {
    if (cfg->page_size != kPageSize) return MLRA_ERR_UNSUPPORTED;
    if (num_pages < 1 || num_pages > (int64_t(1) << 31) / kPageSize) return MLRA_ERR_INVALID_ARG;
  }
  if (!aligned(kv_cache, 16) || !aligned(q_abs, 16) || !aligned(q_rope, 16) ||
      !aligned(seqlens, 4) || (page_table && !aligned(page_table, 4)))
    return MLRA_ERR_ALIGNMENT;
  Grid g;
  st = plan_grid(*cfg, &g);
  if (st != MLRA_OK) return st;
  const WsLayout L = layout_for(*cfg, batch, g);
  if (workspace_bytes < L.total) return MLRA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  const int64_t cap64 = page_table ? int64_t(max_pages) * kPageSize : int64_t(max_pages);
  if (cap64 > (int64_t(1) << 30)) return MLRA_ERR_INVALID_ARG;
  const int cap = (int)cap64;
  cudaError_t e = launch_plan(seqlens, batch, cap, g.ctas_per_group, workspace, L, s);
  if (e != cudaSuccess) return MLRA_ERR_CUDA;
  if (batch == 0) return MLRA_OK;
  DecodeArgs a;
  a.cfg = *cfg;
  a.q_abs = q_abs;
  a.q_rope = q_rope;
  a.kv_cache = kv_cache;
  a.num_pages = page_table ? num_pages : 0;
  a.page_table = page_table;
  a.max_pages = max_pages;
  a.cap = cap;
  a.seqlens = seqlens;
  a.batch = batch;
  a.ws = workspace;
  a.L = L;
  a.ctas_per_group = g.ctas_per_group;
  a.n_groups = g.n_groups;
  a.stall_tile = test_stall_tile();
  e = (g.kind == 1) ? launch_decode_tc(a, s) : launch_decode_simt(a, s);
  return from_cuda(e);
}

mlra_status_t mlra_splitkv_combine(const mlra_config_t* cfg, const void* workspace,
                                   size_t workspace_bytes, int32_t batch, float* o_latent,
                                   float* lse, mlra_stream_t stream) {
  mlra_status_t st = check_cfg(cfg);
  if (st != MLRA_OK) return st;
  if (batch < 0 || !workspace) return MLRA_ERR_INVALID_ARG;
  if (batch == 0) return MLRA_OK;
  if (!o_latent) return MLRA_ERR_INVALID_ARG;
  Grid g;
  st = plan_grid(*cfg, &g);
  if (st != MLRA_OK) return st;
  const WsLayout L = layout_for(*cfg, batch, g);
  if (workspace_bytes < L.total) return MLRA_ERR_WORKSPACE;
  return from_cuda(launch_combine(*cfg, workspace, L, batch, o_latent, lse, (cudaStream_t)stream));
}

mlra_status_t mlra_out_proj(const mlra_config_t* cfg, const float* o_latent, const void* w_uv,
                            float* out, int32_t batch, mlra_stream_t stream) {
  mlra_status_t st = check_cfg(cfg);
  if (st != MLRA_OK) return st;
  if (batch < 0) return MLRA_ERR_INVALID_ARG;
  if (batch == 0) return MLRA_OK;
  if (!o_latent || !w_uv || !out) return MLRA_ERR_INVALID_ARG;
  if (!aligned(w_uv, 16) || !aligned(o_latent, 4) || !aligned(out, 4)) return MLRA_ERR_ALIGNMENT;
  if (use_proj_tc(*cfg) && aligned(o_latent, 16)) {
    WsLayout none{};
    cudaError_t e = launch_out_proj_tc(*cfg, o_latent, nullptr, none, nullptr, nullptr, w_uv, out,
                                       batch, (cudaStream_t)stream);
    if (e != cudaErrorNotSupported) return from_cuda(e);
  }
  return from_cuda(launch_out_proj(*cfg, o_latent, w_uv, out, batch, (cudaStream_t)stream));
}

mlra_status_t mlra_combine_out_proj(const mlra_config_t* cfg, const void* workspace,
                                    size_t workspace_bytes, int32_t batch, const void* w_uv,
                                    float* out, float* o_latent, float* lse,
                                    mlra_stream_t stream) {
  mlra_status_t st = check_cfg(cfg);
  if (st != MLRA_OK) return st;
  if (batch < 0 || !workspace) return MLRA_ERR_INVALID_ARG;
  if (batch == 0) return MLRA_OK;
  if (!w_uv || !out) return MLRA_ERR_INVALID_ARG;
  if (!aligned(w_uv, 16) || !aligned(out, 4) || (o_latent && !aligned(o_latent, 4)) ||
      (lse && !aligned(lse, 4)))
    return MLRA_ERR_ALIGNMENT;
  Grid g;
  st = plan_grid(*cfg, &g);
  if (st != MLRA_OK) return st;
  const WsLayout L = layout_for(*cfg, batch, g);
  if (workspace_bytes < L.total) return MLRA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  if (use_proj_tc(*cfg) && (!o_latent || aligned(o_latent, 16))) {
    cudaError_t e = launch_out_proj_tc(*cfg, nullptr, workspace, L, o_latent, lse,
                                       w_uv, out, batch, s);
    if (e != cudaErrorNotSupported) return from_cuda(e);
  }
  if (!o_latent) return MLRA_ERR_UNSUPPORTED;
  cudaError_t e = launch_combine(*cfg, workspace, L, batch, o_latent, lse, s);
  if (e != cudaSuccess) return MLRA_ERR_CUDA;
  return from_cuda(launch_out_proj(*cfg, o_latent, w_uv, out, batch, s));
}

mlra_status_t mlra_step_workspace_size(const mlra_config_t* cfg, int32_t batch, size_t* bytes) {
  mlra_status_t st = check_cfg(cfg);
  if (st != MLRA_OK) return st;
  if (batch < 0 || !bytes) return MLRA_ERR_INVALID_ARG;
  Grid g;
  st = plan_grid(*cfg, &g);
  if (st != MLRA_OK) return st;
  *bytes = step_layout(*cfg, batch, g).total;
  return MLRA_OK;
}

mlra_status_t mlra_decode_step(const mlra_config_t* cfg, const void* q_nope, const void* q_rope,
                               const int32_t* seqlens, int32_t batch, const void* w_uk,
                               const void* w_uv, const void* kv_cache, int64_t num_pages,
                               const int32_t* page_table, int32_t max_pages, float* out,
                               int32_t host_io, void* workspace, size_t workspace_bytes,
                               mlra_stream_t stream) {
  mlra_status_t st = check_cfg(cfg);
  if (st != MLRA_OK) return st;
  if (batch < 0 || !workspace || (host_io != 0 && host_io != 1)) return MLRA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MLRA_ERR_WORKSPACE;
  if (batch == 0) return MLRA_OK;
  if (!q_nope || !q_rope || !seqlens || !w_uk || !w_uv || !kv_cache || !out)
    return MLRA_ERR_INVALID_ARG;
  Grid g;
  st = plan_grid(*cfg, &g);
  if (st != MLRA_OK) return st;
  StepCall c;
  c.cfg = *cfg;
  c.q_nope = q_nope;
  c.q_rope = q_rope;
  c.seqlens = seqlens;
  c.batch = batch;
  c.w_uk = w_uk;
  c.w_uv = w_uv;
  c.kv_cache = kv_cache;
  c.num_pages = num_pages;
  c.page_table = page_table;
  c.max_pages = max_pages;
  c.out = out;
  c.host_io = host_io;
  c.workspace = workspace;
  c.workspace_bytes = workspace_bytes;
  c.S = step_layout(*cfg, batch, g);
  if (workspace_bytes < c.S.total) return MLRA_ERR_WORKSPACE;
  resolve_step(&c);
  return run_step(c, (cudaStream_t)stream);
}

mlra_status_t mlra_release_step_graphs(void) {
  std::lock_guard<std::mutex> lock(g_step_mu);
  mlra_status_t st = MLRA_OK;
  for (int i = 0; i < g_step_n; ++i) {
    if (g_step_graphs[i].state == 2 && cudaGraphExecDestroy(g_step_graphs[i].exec) != cudaSuccess)
      st = MLRA_ERR_CUDA;
    g_step_graphs[i] = StepGraph{};
  }
  g_step_n = 0;
  (void)cudaGetLastError();
  return st;
}

mlra_status_t mlra_cache_append(const mlra_config_t* cfg, const void* c_new,
                                const void* k_rope_new, const float* rms_gamma, float alpha_kv,
                                float rms_eps, float rope_theta, void* kv_cache,
                                int64_t num_pages, const int32_t* page_table, int32_t max_pages,
                                const int32_t* positions, int32_t batch, int32_t* device_status,
                                mlra_stream_t stream) {
  mlra_status_t st = check_cfg(cfg);
  if (st != MLRA_OK) return st;
  if (batch < 0) return MLRA_ERR_INVALID_ARG;
  if (batch == 0) return MLRA_OK;
  if (!c_new || !k_rope_new || !rms_gamma || !kv_cache || !positions) return MLRA_ERR_INVALID_ARG;
  if (cfg->d_r % 2 != 0 || max_pages < 1) return MLRA_ERR_INVALID_ARG;
  if (!(rope_theta > 0.f) || !(rms_eps >= 0.f) || !(alpha_kv == alpha_kv)) return MLRA_ERR_INVALID_ARG;
  if (page_table) {
    if (cfg->page_size != kPageSize) return MLRA_ERR_UNSUPPORTED;
    if (num_pages < 1 || num_pages > (int64_t(1) << 31) / kPageSize) return MLRA_ERR_INVALID_ARG;
  }
  const uintptr_t el = cfg->dtype == MLRA_BF16 ? 2 : 4;
  if (!aligned(c_new, el) || !aligned(k_rope_new, el) || !aligned(kv_cache, el) ||
      !aligned(rms_gamma, 4) || !aligned(positions, 4) || (page_table && !aligned(page_table, 4)) ||
      (device_status && !aligned(device_status, 4)))
    return MLRA_ERR_ALIGNMENT;
  const int64_t cap64 = page_table ? int64_t(max_pages) * kPageSize : int64_t(max_pages);
  if (cap64 > (int64_t(1) << 30)) return MLRA_ERR_INVALID_ARG;
  return from_cuda(launch_cache_append(*cfg, c_new, k_rope_new, rms_gamma, alpha_kv, rms_eps,
                                       double(rope_theta), kv_cache, page_table ? num_pages : 0,
                                       page_table, max_pages, int(cap64), positions, batch,
                                       device_status, (cudaStream_t)stream));
}

mlra_status_t mlra_get_device_error(const void* workspace, size_t workspace_bytes,
                                    int32_t* device_status, mlra_stream_t stream) {
  if (!workspace || !device_status || workspace_bytes < sizeof(WsHeader))
    return MLRA_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  int32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return MLRA_ERR_CUDA;
  *device_status = v;
  if (v != 0) {
    e = cudaMemsetAsync(const_cast<void*>(workspace), 0, sizeof(int32_t), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return MLRA_ERR_CUDA;
  }
  return MLRA_OK;
}

}  // extern "C"
