// Host-side entry points of the kernel files, used by the C ABI (mlra_api.cu).
// Nothing here is part of the C ABI (include/mlra.h).
#pragma once

#include "mlra_internal.cuh"

namespace mlra {

// Dispatch entry points of the individual kernel files (host side).
cudaError_t launch_plan(const int32_t* seqlens, int batch, int cap, int ctas_per_group, void* ws,
                        const WsLayout& L, cudaStream_t st);
// q_abs = alpha * W_uk q_nope (alpha = 1: the plain absorption).
cudaError_t launch_absorb(const mlra_config_t& c, const void* q_nope, const void* w_uk,
                          float* q_abs, int batch, float alpha, cudaStream_t st);
cudaError_t launch_combine(const mlra_config_t& c, const void* ws, const WsLayout& L, int batch,
                           float* o_latent, float* lse, cudaStream_t st);
cudaError_t launch_out_proj(const mlra_config_t& c, const float* o_latent, const void* w_uv,
                            float* out, int batch, cudaStream_t st);

// Copies of up to three byte ranges in one launch, each source being host
// memory mapped into the device address space (k_small.cu).
struct StageCopy {
  const void* src;
  void* dst;
  size_t bytes;
};
cudaError_t launch_stage(const StageCopy* copies, int n, cudaStream_t st);

// Query side of the step (k_cache.cu): q_rope_out = RoPE(alpha * q_rope) at
// each sequence's position, in the storage dtype.
cudaError_t launch_query_rope(const mlra_config_t& c, const void* q_rope, const int32_t* positions,
                              float alpha, double theta, void* q_rope_out, int batch,
                              cudaStream_t st);

// Cache write (k_cache.cu).
cudaError_t launch_cache_append(const mlra_config_t& c, const void* c_new, const void* k_rope_new,
                                const float* gamma, float alpha_kv, float eps, double theta,
                                void* kv_cache, int64_t num_pages, const int32_t* page_table,
                                int max_pages, int cap, const int32_t* positions, int batch,
                                int32_t* status, cudaStream_t st);

// Tensor-core absorption and output projection (bf16, d_h = 128).
bool proj_tc_supported(const mlra_config_t& c);
cudaError_t launch_absorb_tc(const mlra_config_t& c, const void* q_nope, const void* w_uk,
                             float* q_abs, int batch, float alpha, cudaStream_t st);
cudaError_t launch_out_proj_tc(const mlra_config_t& c, const float* o_latent_in, const void* ws,
                               const WsLayout& L, float* o_latent_out,
                               float* lse_out, const void* w_uv, float* out, int batch,
                               cudaStream_t st);

// fp32 SIMT decode (any supported shape / dtype).
bool simt_supported(const mlra_config_t& c);
void simt_grid(const mlra_config_t& c, int num_sms, int* n_groups, int* ctas_per_group);
cudaError_t launch_decode_simt(const DecodeArgs& a, cudaStream_t st);

// Tensor-core decode (tcgen05 / TMEM / TMA), bf16 cache.
bool tc_supported(const mlra_config_t& c);
void tc_grid(const mlra_config_t& c, int num_sms, int* n_groups, int* ctas_per_group);
cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t st);

}  // namespace mlra
