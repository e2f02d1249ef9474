// noalloc.cu -- hpa_decode_noalloc: one decode step (plan + run) whose
// scratch lives in a fixed, library-owned device array instead of a
// caller-allocated workspace.
//
// Who needs it: callers that cannot allocate device memory at the point where
// they run a decode step -- for example code that runs inside a memory pool
// that must not grow after start-up, a caller whose allocator is owned by
// another framework and is not reachable from where the step is issued, or a
// plain C host program that has no allocator of its own and must not call
// cudaMalloc on its hot path.  Such a caller still passes its inputs and
// outputs; only the plan, the split partials and the arrival counters move
// into this array.
//
// The array is HPA_NOALLOC_SCRATCH_BYTES (16 MiB) per GPU that loads the
// library and stays allocated until the process exits.  All calls on a
// device share it and it keeps the previous call's contents: the plan kernel
// rewrites every field the run reads and zeroes the arrival counters on each
// call, so stale contents never leak into a result, but two calls whose work
// overlaps on the GPU (different streams, no ordering between them) race on
// the same array and produce garbage.
#include <mutex>

#include "hpa_common.cuh"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[HPA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};

// Device address of the scratch array and the SM count for the current
// device, looked up once per device with that device current.  In host code
// `g_noalloc_scratch` is only a host-side stand-in; the kernels must be given
// the address cudaGetSymbolAddress returns.
hpa_status device_setup(int* dev_out, void** ptr_out, int* sms_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    hpa::set_cuda_error(e, "hpa_decode_noalloc cudaGetDevice");
    return HPA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return HPA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || !ptr) {
      hpa::set_cuda_error(e, "hpa_decode_noalloc cudaGetSymbolAddress");
      return HPA_ERR_CUDA;
    }
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess || sms <= 0) {
      hpa::set_cuda_error(e, "hpa_decode_noalloc cudaDeviceGetAttribute");
      return HPA_ERR_CUDA;
    }
    g_num_sms[dev] = sms;
    g_scratch_ptr[dev] = ptr;
  }
  *dev_out = dev;
  *ptr_out = g_scratch_ptr[dev];
  *sms_out = g_num_sms[dev];
  return HPA_OK;
}

}  // namespace

extern "C" hpa_status hpa_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                         const float* k_scale, const float* v_scale,
                                         hpa_kv_dtype kv_dtype, const int32_t* page_table,
                                         int pt_stride, int num_pages, const int32_t* seq_lens,
                                         void* out, hpa_out_dtype out_dtype, int batch,
                                         int num_q_heads, int num_kv_heads, int head_dim,
                                         float softmax_scale, int num_ctas, void* stream) {
  // Everything hpa_decode_run would reject is rejected here too, before the
  // plan is enqueued, so a bad call enqueues nothing.
  if (num_ctas < 0 || !seq_lens || !q || !k_cache || !v_cache || !page_table || !out)
    return HPA_ERR_INVALID_ARG;
  if (batch <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || pt_stride <= 0 || num_pages <= 0 ||
      num_q_heads % num_kv_heads)
    return HPA_ERR_INVALID_ARG;
  if ((kv_dtype != HPA_KV_BF16 && kv_dtype != HPA_KV_FP8_E4M3) ||
      (out_dtype != HPA_OUT_BF16 && out_dtype != HPA_OUT_F32))
    return HPA_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || softmax_scale == INFINITY) return HPA_ERR_INVALID_ARG;
  if (kv_dtype == HPA_KV_FP8_E4M3 && (!k_scale || !v_scale)) return HPA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache)) & 15 ||
      (reinterpret_cast<uintptr_t>(q) & 15) || (reinterpret_cast<uintptr_t>(out) & 3))
    return HPA_ERR_INVALID_ARG;
  {
    const int G = num_q_heads / num_kv_heads;
    if (G > 32) return HPA_ERR_UNSUPPORTED;  // a kv head's rows fill at most four MMA n-tiles
    if (head_dim != 64 && head_dim != 128) return HPA_ERR_UNSUPPORTED;
    if (kv_dtype == HPA_KV_FP8_E4M3 && head_dim != 128) return HPA_ERR_UNSUPPORTED;
    if ((long long)num_pages * num_kv_heads * 64 > 0x7fffffffLL) return HPA_ERR_UNSUPPORTED;
  }
  // Size check first, on the host, so an oversized request is refused before
  // any CUDA call.
  if (num_ctas > 0) {
    const size_t need =
        hpa_decode_workspace_size(HPA_PLAN_DYNAMIC, batch, num_kv_heads, num_q_heads, head_dim,
                                  num_ctas);
    if (need == 0) return HPA_ERR_INVALID_ARG;
    if (need > HPA_NOALLOC_SCRATCH_BYTES) return HPA_ERR_WORKSPACE;
  }
  int dev = 0, sms = 0;
  void* scratch = nullptr;
  hpa_status st = device_setup(&dev, &scratch, &sms);
  if (st != HPA_OK) return st;
  const int ctas = num_ctas > 0 ? num_ctas : sms;
  const size_t need = hpa_decode_workspace_size(HPA_PLAN_DYNAMIC, batch, num_kv_heads, num_q_heads,
                                                head_dim, ctas);
  if (need == 0) return HPA_ERR_INVALID_ARG;
  if (need > HPA_NOALLOC_SCRATCH_BYTES) return HPA_ERR_WORKSPACE;
  // Up to kMaxFusedBatch (512) sequences the plan is made inside the decode
  // kernel (the static array starts zero-filled, and every dynamic run leaves
  // its run-time counters at zero); larger batches take the plan kernel.
  if (batch <= hpa::kMaxFusedBatch)
    return hpa_decode_step(seq_lens, q, k_cache, v_cache, k_scale, v_scale, kv_dtype, page_table,
                           pt_stride, num_pages, out, out_dtype, batch, 1, num_q_heads,
                           num_kv_heads, head_dim, softmax_scale, ctas, scratch,
                           HPA_NOALLOC_SCRATCH_BYTES, stream);
  // (the plan the in-kernel plan would make: its cost weights depend on the
  // cache type)
  int grid = 0;
  st = hpa_decode_plan_shape(seq_lens, batch, num_kv_heads, num_q_heads, head_dim, pt_stride,
                             HPA_PLAN_DYNAMIC, ctas, 0, HPA_TAIL_DEN_DEFAULT,
                             HPA_TAIL_CHUNKS_DEFAULT, HPA_TAIL_MIN_DEFAULT, HPA_COST_UNIT_DEFAULT,
                             kv_dtype == HPA_KV_FP8_E4M3 ? HPA_COST_END_DEFAULT_FP8
                                                         : HPA_COST_END_DEFAULT,
                             scratch, HPA_NOALLOC_SCRATCH_BYTES, &grid, stream);
  if (st != HPA_OK) return st;
  return hpa_decode_run(q, k_cache, v_cache, k_scale, v_scale, kv_dtype, page_table, pt_stride,
                        num_pages, out, out_dtype, batch, num_q_heads, num_kv_heads, head_dim,
                        softmax_scale, HPA_PLAN_DYNAMIC, grid, scratch,
                        HPA_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" hpa_status hpa_noalloc_read_status(int32_t* status_out, int clear, void* stream) {
  if (!status_out) return HPA_ERR_INVALID_ARG;
  int dev = 0, sms = 0;
  void* scratch = nullptr;
  hpa_status st = device_setup(&dev, &scratch, &sms);
  if (st != HPA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* word = static_cast<int32_t*>(scratch) + hpa::kHdrStatus;
  cudaError_t e = cudaMemcpyAsync(status_out, word, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess && clear) e = cudaMemsetAsync(word, 0, sizeof(int32_t), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    hpa::set_cuda_error(e, "hpa_noalloc_read_status");
    return HPA_ERR_CUDA;
  }
  return HPA_OK;
}
