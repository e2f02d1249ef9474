// prologue.cu -- fused RMSNorm + RoPE + KV write for the new decode token
// (hpa_kv_prologue).
//
// The method (bitbyai.com "vLLM x HPC-Ops", Attention Backend): RoPE,
// query-key normalisation and the KV-cache write are fused into one prologue,
// saving launches and HBM round trips.  One CTA per sequence; one warp per
// head row (q heads, then k heads, then v heads); the row arithmetic (and its
// precision) is in prologue_math.cuh, shared with the decode kernel's fused
// prologue.
#include <cmath>

#include <cuda_bf16.h>

#include "hpa_common.cuh"
#include "prologue_math.cuh"

namespace hpa {
namespace {

constexpr int kPrologueWarps = 8;

struct PrologueParams {
  const __nv_bfloat16* q_raw;
  const __nv_bfloat16* k_raw;
  const __nv_bfloat16* v_raw;
  const float* q_gamma;
  const float* k_gamma;
  float eps;
  double log2_theta;
  const int32_t* positions;
  const int32_t* page_table;
  int pt_stride, num_pages;
  __nv_bfloat16* k_cache;
  __nv_bfloat16* v_cache;
  __nv_bfloat16* q_out;
  int Hq, Hkv;
  int32_t* status;
};

template <int D>
__global__ void __launch_bounds__(kPrologueWarps * 32) prologue_kernel(const PrologueParams p) {
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  const int pos = p.positions[b];

  RopeLane<D> rope;
  rope.init(pos, lane, p.log2_theta);

  // destination slot of the new K/V row
  long long slot_row = -1;
  if (pos >= 0 && pos / kPageSize < p.pt_stride) {
    const int page = p.page_table[(long long)b * p.pt_stride + pos / kPageSize];
    if (page >= 0 && page < p.num_pages) slot_row = (long long)page * p.Hkv * kPageSize + pos % kPageSize;
  }
  if (slot_row < 0 && threadIdx.x == 0 && p.status) atomicOr(p.status, HPA_DEVICE_BAD_POSITION);

  const int rows = p.Hq + 2 * p.Hkv;
  for (int row = warp; row < rows; row += kPrologueWarps) {
    const __nv_bfloat16* src;
    __nv_bfloat16* dst;
    const float* gamma = nullptr;
    if (row < p.Hq) {
      src = p.q_raw + ((long long)b * p.Hq + row) * D;
      dst = p.q_out + ((long long)b * p.Hq + row) * D;
      gamma = p.q_gamma;
    } else if (row < p.Hq + p.Hkv) {
      const int g = row - p.Hq;
      src = p.k_raw + ((long long)b * p.Hkv + g) * D;
      dst = slot_row < 0 ? nullptr : p.k_cache + (slot_row + (long long)g * kPageSize) * D;
      gamma = p.k_gamma;
    } else {
      const int g = row - p.Hq - p.Hkv;
      src = p.v_raw + ((long long)b * p.Hkv + g) * D;
      dst = slot_row < 0 ? nullptr : p.v_cache + (slot_row + (long long)g * kPageSize) * D;
    }
    if (!gamma) {  // V: bit copy into the slot
      if (dst)
        for (int i = lane; i < D; i += 32) dst[i] = src[i];
      continue;
    }
    norm_rope_row<D>(src, dst, nullptr, gamma, p.eps, rope, lane);
  }
  pdl_trigger();
}

}  // namespace
}  // namespace hpa

using namespace hpa;

extern "C" hpa_status hpa_kv_prologue(const void* q_raw, const void* k_raw, const void* v_raw,
                                      const float* q_gamma, const float* k_gamma, float eps,
                                      float rope_theta, const int32_t* positions,
                                      const int32_t* page_table, int pt_stride, void* k_cache,
                                      void* v_cache, void* q_out, int batch, int num_q_heads,
                                      int num_kv_heads, int head_dim, int num_pages,
                                      int32_t* status, void* stream) {
  if (!q_raw || !k_raw || !v_raw || !q_gamma || !k_gamma || !positions || !page_table ||
      !k_cache || !v_cache || !q_out)
    return HPA_ERR_INVALID_ARG;
  if (batch <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || pt_stride <= 0 || num_pages <= 0)
    return HPA_ERR_INVALID_ARG;
  if (num_q_heads % num_kv_heads) return HPA_ERR_INVALID_ARG;
  if (!(eps >= 0.f) || !(rope_theta > 0.f) || !std::isfinite(eps) || !std::isfinite(rope_theta))
    return HPA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return HPA_ERR_UNSUPPORTED;
  if ((long long)num_pages * num_kv_heads * kPageSize * head_dim > (1LL << 62))
    return HPA_ERR_UNSUPPORTED;

  PrologueParams p;
  p.q_raw = static_cast<const __nv_bfloat16*>(q_raw);
  p.k_raw = static_cast<const __nv_bfloat16*>(k_raw);
  p.v_raw = static_cast<const __nv_bfloat16*>(v_raw);
  p.q_gamma = q_gamma;
  p.k_gamma = k_gamma;
  p.eps = eps;
  p.log2_theta = std::log2((double)rope_theta);
  p.positions = positions;
  p.page_table = page_table;
  p.pt_stride = pt_stride;
  p.num_pages = num_pages;
  p.k_cache = static_cast<__nv_bfloat16*>(k_cache);
  p.v_cache = static_cast<__nv_bfloat16*>(v_cache);
  p.q_out = static_cast<__nv_bfloat16*>(q_out);
  p.Hq = num_q_heads;
  p.Hkv = num_kv_heads;
  p.status = status;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(batch);
  cfg.blockDim = dim3(kPrologueWarps * 32);
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = head_dim == 128 ? cudaLaunchKernelEx(&cfg, prologue_kernel<128>, p)
                                  : cudaLaunchKernelEx(&cfg, prologue_kernel<64>, p);
  if (e != cudaSuccess) {
    set_cuda_error(e, "hpa_kv_prologue launch");
    return HPA_ERR_CUDA;
  }
  return HPA_OK;
}
