// merge_states.cu -- log-sum-exp merge of attention states computed over
// disjoint parts of the same keys (hpa_merge_states).
//
// The split-KV decode of xiaodao.ai "HPC-Ops TPOT -48.8%" (Attention section)
// cuts a sequence's KV into pieces and recombines the pieces' partial results;
// inside one GPU the decode kernel and its merge kernel do that.  This call is
// the same recombination for states that were computed apart: by decode steps
// over different page ranges of the same sequences (a sequence whose KV is
// spread over the GPUs of a tensor-parallel group, openai-hub.com news/688:
// cross-GPU communication in tensor/expert-parallel serving), or over a
// shared prefix and a private suffix.  State i of a row is its normalised
// output o_i and its log-sum-exp lse_i = log sum_j exp(scale q.k_j) over the
// part's keys; the merged row is
//
//     L = log sum_i exp(lse_i),   o = sum_i exp(lse_i - L) o_i,
//
// evaluated as M = max_i lse_i, w_i = exp(lse_i - M), lam = sum_i w_i,
// o = sum_i (w_i / lam) o_i (folded in index order), L = M + log lam.
//
// One warp per row: lane i fetches lse_i while every lane loads its D/32
// elements of all the states' rows (one round trip to memory); the weights
// come from two warp reductions, and a state with lse = -inf is left out of
// the sum (its row may hold anything).  The loads are plain (coherent) global
// loads, neither TMA nor the read-only path, so a state may live in a peer
// GPU's memory mapped into this context.
#include <algorithm>
#include <atomic>
#include <cmath>

#include <cuda_bf16.h>

#include "hpa_common.cuh"

namespace hpa {
namespace {

constexpr int kMaxStates = 16;
constexpr int kStateWarps = 8;

struct StateParams {
  const float* o[kMaxStates];
  const float* lse[kMaxStates];
  int n;
  long long rows;
  void* out;
  float* lse_out;
};

template <int D, bool OUT_F32>
__global__ void __launch_bounds__(kStateWarps * 32) merge_states_kernel(const StateParams p) {
  constexpr int kVec = D / 32;
  pdl_wait();  // the states may come from the kernel before this one
  const int lane = threadIdx.x & 31;
  const long long stride = (long long)gridDim.x * kStateWarps;
  for (long long r = (long long)blockIdx.x * kStateWarps + (threadIdx.x >> 5); r < p.rows;
       r += stride) {
    // the states' rows and log-sum-exps are loaded together (one round trip)
    const float li = lane < p.n ? p.lse[lane][r] : -INFINITY;
    float x[kMaxStates][kVec];
#pragma unroll
    for (int i = 0; i < kMaxStates; ++i) {
      const float* src = p.o[i < p.n ? i : 0] + r * D + lane * kVec;
      if constexpr (kVec == 4) {
        const float4 a = i < p.n ? *reinterpret_cast<const float4*>(src)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
        x[i][0] = a.x; x[i][1] = a.y; x[i][2] = a.z; x[i][3] = a.w;
      } else {
        const float2 a = i < p.n ? *reinterpret_cast<const float2*>(src) : make_float2(0.f, 0.f);
        x[i][0] = a.x; x[i][1] = a.y;
      }
    }
    float M = li;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float w = (li == -INFINITY) ? 0.f : expf(li - M);
    float lam = w;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) lam += __shfl_xor_sync(0xffffffffu, lam, off);
    float o[kVec];
#pragma unroll
    for (int v = 0; v < kVec; ++v) o[v] = 0.f;
    if (lam > 0.f) {  // warp-uniform
      const float inv = 1.f / lam;
#pragma unroll
      for (int i = 0; i < kMaxStates; ++i) {
        const float wi = __shfl_sync(0xffffffffu, w, i) * inv;
        if (i < p.n && wi != 0.f) {  // an empty state's row is never used
#pragma unroll
          for (int v = 0; v < kVec; ++v) o[v] = fmaf(wi, x[i][v], o[v]);
        }
      }
    }
    if constexpr (OUT_F32) {
      float* dst = reinterpret_cast<float*>(p.out) + r * D + lane * kVec;
      if constexpr (kVec == 4) *reinterpret_cast<float4*>(dst) = make_float4(o[0], o[1], o[2], o[3]);
      else *reinterpret_cast<float2*>(dst) = make_float2(o[0], o[1]);
    } else {
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + r * D + lane * kVec;
      if constexpr (kVec == 4) *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]));
      else *reinterpret_cast<uint32_t*>(dst) = pack_bf16(o[0], o[1]);
    }
    if (p.lse_out && lane == 0) p.lse_out[r] = lam > 0.f ? M + logf(lam) : -INFINITY;
  }
  pdl_trigger();
}

int device_sms() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  int n = cache[dev].load();
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev].store(n);
  }
  return n;
}

// Whether this device's kernels can reach `ptr`, as far as the driver can
// tell: memory of the current device, managed memory, pinned host memory
// mapped into the address space, or memory of a peer device this one can
// access (the caller must have enabled that access).  A pageable host pointer
// or an address the driver does not know is refused.  Pointers found
// reachable are remembered per host thread (the same state buffers come back
// every step), so a step pays the driver query once.
hpa_status check_reachable(const void* ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    set_cuda_error(e, "hpa_merge_states cudaGetDevice");
    return HPA_ERR_CUDA;
  }
  constexpr int kSeen = 64;
  thread_local const void* seen[kSeen] = {};
  thread_local int seen_dev[kSeen] = {};
  thread_local int next = 0;
  for (int i = 0; i < kSeen; ++i)
    if (seen[i] == ptr && seen_dev[i] == dev) return HPA_OK;
  cudaPointerAttributes a;
  e = cudaPointerGetAttributes(&a, ptr);
  if (e != cudaSuccess) {
    cudaGetLastError();
    set_cuda_error(e, "hpa_merge_states cudaPointerGetAttributes");
    return HPA_ERR_CUDA;
  }
  bool ok = false;
  if (a.type == cudaMemoryTypeManaged) {
    ok = true;
  } else if (a.type == cudaMemoryTypeHost) {
    ok = a.devicePointer == ptr;  // mapped pinned memory at the same address
  } else if (a.type == cudaMemoryTypeDevice) {
    int can = a.device == dev;
    if (!can && cudaDeviceCanAccessPeer(&can, dev, a.device) != cudaSuccess) {
      cudaGetLastError();
      can = 0;
    }
    ok = can != 0;
  }
  if (!ok) return HPA_ERR_INVALID_ARG;
  seen[next] = ptr;
  seen_dev[next] = dev;
  next = (next + 1) % kSeen;
  return HPA_OK;
}

}  // namespace
}  // namespace hpa

extern "C" hpa_status hpa_merge_states(const float* const* o_parts, const float* const* lse_parts,
                                       int num_states, long long rows, int head_dim, void* out,
                                       hpa_out_dtype out_dtype, float* lse_out, void* stream) {
  using namespace hpa;
  if (!o_parts || !lse_parts || !out) return HPA_ERR_INVALID_ARG;
  if (num_states < 1 || rows < 0) return HPA_ERR_INVALID_ARG;
  if (num_states > kMaxStates) return HPA_ERR_UNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return HPA_ERR_UNSUPPORTED;
  if (out_dtype != HPA_OUT_BF16 && out_dtype != HPA_OUT_F32) return HPA_ERR_INVALID_ARG;
  if (rows > (1LL << 40)) return HPA_ERR_UNSUPPORTED;
  StateParams p = {};
  for (int i = 0; i < num_states; ++i) {
    if (!o_parts[i] || !lse_parts[i]) return HPA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(o_parts[i]) & 15) || (reinterpret_cast<uintptr_t>(lse_parts[i]) & 3))
      return HPA_ERR_INVALID_ARG;
    p.o[i] = o_parts[i];
    p.lse[i] = lse_parts[i];
  }
  const bool f32 = out_dtype == HPA_OUT_F32;
  if (reinterpret_cast<uintptr_t>(out) & (f32 ? 15 : 7)) return HPA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(lse_out) & 3) return HPA_ERR_INVALID_ARG;
  if (rows == 0) return HPA_OK;
  // every buffer must be reachable from this device before anything is
  // enqueued (a pageable host pointer would fault the kernel)
  for (int i = 0; i < num_states; ++i)
    for (const void* q : {static_cast<const void*>(o_parts[i]), static_cast<const void*>(lse_parts[i])}) {
      const hpa_status st = check_reachable(q);
      if (st != HPA_OK) return st;
    }
  for (const void* q : {static_cast<const void*>(out), static_cast<const void*>(lse_out)}) {
    if (!q) continue;
    const hpa_status st = check_reachable(q);
    if (st != HPA_OK) return st;
  }
  p.n = num_states;
  p.rows = rows;
  p.out = out;
  p.lse_out = lse_out;

  const int sms = device_sms();
  const long long want = (rows + kStateWarps - 1) / kStateWarps;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)std::min<long long>(want, (long long)std::max(1, sms) * 8));
  cfg.blockDim = dim3(kStateWarps * 32);
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (head_dim == 128)
    e = f32 ? cudaLaunchKernelEx(&cfg, merge_states_kernel<128, true>, p)
            : cudaLaunchKernelEx(&cfg, merge_states_kernel<128, false>, p);
  else
    e = f32 ? cudaLaunchKernelEx(&cfg, merge_states_kernel<64, true>, p)
            : cudaLaunchKernelEx(&cfg, merge_states_kernel<64, false>, p);
  if (e != cudaSuccess) {
    set_cuda_error(e, "hpa_merge_states launch");
    return HPA_ERR_CUDA;
  }
  return HPA_OK;
}
