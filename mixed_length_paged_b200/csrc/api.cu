// api.cu -- host-only entry points of libhpa.so: status strings, version,
// workspace sizing and layout, default CTA count, status readback.
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "hpa_common.cuh"

namespace hpa {

static thread_local char g_last_error[256] = "";

void set_cuda_error(cudaError_t e, const char* where) {
  std::snprintf(g_last_error, sizeof g_last_error, "%s: %s (%s)", where, cudaGetErrorName(e),
                cudaGetErrorString(e));
}

}  // namespace hpa

using namespace hpa;

extern "C" const char* hpa_status_string(hpa_status s) {
  switch (s) {
    case HPA_OK: return "HPA_OK";
    case HPA_ERR_INVALID_ARG: return "HPA_ERR_INVALID_ARG";
    case HPA_ERR_UNSUPPORTED: return "HPA_ERR_UNSUPPORTED";
    case HPA_ERR_WORKSPACE: return "HPA_ERR_WORKSPACE";
    case HPA_ERR_CUDA: return "HPA_ERR_CUDA";
  }
  return "HPA_ERR_UNKNOWN";
}

extern "C" const char* hpa_last_cuda_error(void) { return g_last_error; }

extern "C" int hpa_version(void) { return 100; }

#ifndef HPA_CTAS_PER_SM
#define HPA_CTAS_PER_SM 2
#endif

extern "C" int hpa_default_num_ctas(int device) {
  // HPA_NUM_CTAS (a decimal count, 1 .. 65536) overrides the device default
  if (const char* env = std::getenv("HPA_NUM_CTAS")) {
    char* end = nullptr;
    const long v = std::strtol(env, &end, 10);
    if (end != env && *end == '\0' && v >= 1 && v <= 65536) return (int)v;
  }
  int n = 0;
  cudaError_t e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device);
  if (e != cudaSuccess) {
    set_cuda_error(e, "hpa_default_num_ctas");
    return -1;
  }
  return n * HPA_CTAS_PER_SM;
}

extern "C" int hpa_decode_num_ctas(int device, int num_q_heads, int num_kv_heads,
                                   int q_tokens) {
  if (num_q_heads <= 0 || num_kv_heads <= 0 || q_tokens <= 0 || num_q_heads % num_kv_heads)
    return -1;
  const long long rows = (long long)(num_q_heads / num_kv_heads) * q_tokens;
  if (rows > 32) return -1;
  // up to 32 query rows per kv head the run kernel runs two CTAs per SM (the
  // two-n-tile kernel splits its warps by n-tile; the four-n-tile kernel
  // then keeps one deposit buffer and two stages)
  return hpa_default_num_ctas(device);
}

extern "C" size_t hpa_decode_workspace_size(hpa_plan_kind kind, int batch, int num_kv_heads,
                                            int num_q_heads, int head_dim, int grid) {
  WsLayout L;
  if (!ws_layout(kind, batch, num_kv_heads, num_q_heads, head_dim, grid, &L)) return 0;
  return L.total;
}

extern "C" hpa_status hpa_workspace_layout(hpa_plan_kind kind, int batch, int num_kv_heads,
                                           int num_q_heads, int head_dim, int grid,
                                           size_t offsets[8]) {
  WsLayout L;
  if (!offsets || !ws_layout(kind, batch, num_kv_heads, num_q_heads, head_dim, grid, &L))
    return HPA_ERR_INVALID_ARG;
  const size_t v[8] = {L.header,   L.lens,    L.tile_start, L.cta_desc,
                       L.seg_desc, L.part_ml, L.part_acc,   L.total};
  std::memcpy(offsets, v, sizeof v);
  return HPA_OK;
}

extern "C" hpa_status hpa_read_status(const void* workspace, int32_t* status_out, void* stream) {
  if (!workspace || !status_out) return HPA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int32_t* src = static_cast<const int32_t*>(workspace) + kHdrStatus;
  cudaError_t e = cudaMemcpyAsync(status_out, src, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    set_cuda_error(e, "hpa_read_status");
    return HPA_ERR_CUDA;
  }
  return HPA_OK;
}

extern "C" hpa_status hpa_read_cta_times(const void* workspace, hpa_plan_kind kind, int batch,
                                         int num_kv_heads, int num_q_heads, int head_dim,
                                         int grid, uint64_t* times_out, void* stream) {
  WsLayout L;
  if (!workspace || !times_out || !ws_layout(kind, batch, num_kv_heads, num_q_heads, head_dim,
                                             grid, &L))
    return HPA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const char* src = static_cast<const char*>(workspace) + L.trace;
  cudaError_t e = cudaMemcpyAsync(times_out, src, size_t(grid) * 4 * sizeof(uint64_t),
                                  cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    set_cuda_error(e, "hpa_read_cta_times");
    return HPA_ERR_CUDA;
  }
  return HPA_OK;
}
