// plan.cu -- per-step tile planner (hpa_decode_plan).
//
// The method (xiaodao.ai "HPC-Ops TPOT -48.8%", Attention section; bitbyai.com
// "vLLM x HPC-Ops", Attention Backend): cut each sequence's live KV into
// 64-token tiles and spread the global task list as evenly as possible over
// persistent CTAs, so a long sequence takes many CTAs and a short one only
// the tiles it has.  The static split-KV schedules the pages compare against
// (fixed split count; fixed split size with the grid sized by the longest
// request) come out of the same kernel so that one run kernel serves all.
//
// One CTA of 1024 threads builds the whole plan on the device from the
// device-side lengths, so a decode step needs no host round trip.  Units are
// (sequence b, kv head g, tile t) in that order; segment s = b * Hkv + g.
#include <algorithm>

#include "hpa_common.cuh"

namespace hpa {
namespace {

constexpr int kPlanThreads = 1024;

struct PlanParams {
  const int32_t* seq_lens;
  int B, Hkv, G, D, capacity;  // capacity = pt_stride * 64 tokens
  int kind, num_ctas, grid;
  long long chunk;             // STATIC_CHUNK: tiles per split
  Ws ws;
};

// Exclusive block-wide prefix sum of one int per thread; *total gets the sum.
__device__ int block_exclusive_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < (kPlanThreads / 32) ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    s_warp[lane] = w;  // inclusive prefix of warp sums
  }
  __syncthreads();
  const int before = (warp > 0 ? s_warp[warp - 1] : 0) + x - v;
  *total = s_warp[kPlanThreads / 32 - 1];
  __syncthreads();
  return before;
}

// Largest b in [0, B) with tile_start[b] * Hkv <= u (u < U).
__device__ int seq_of_unit(const int32_t* tile_start, int B, int Hkv, long long u) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if ((long long)tile_start[mid] * Hkv <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Dynamic plan: CTA holding unit u when U units are spread over P CTAs as
// [floor(cU/P), floor((c+1)U/P)):  the largest c with floor(cU/P) <= u.
__device__ __forceinline__ long long cta_of(long long u, long long U, long long P) {
  return ((u + 1) * P - 1) / U;
}

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(PlanParams p) {
  __shared__ int s_warp[32];
  __shared__ int s_status;
  // The previous step's run kernel may still be reading this workspace.
  pdl_wait();
  const int tid = threadIdx.x;
  if (tid == 0) s_status = 0;
  __syncthreads();

  // 1. clamped lengths, tiles per sequence, exclusive tile prefix sum
  int carry = 0;
  for (int base = 0; base < p.B; base += kPlanThreads) {
    const int b = base + tid;
    int n = 0;
    if (b < p.B) {
      const int L = p.seq_lens[b];
      const int Lc = min(max(L, 0), p.capacity);
      if (Lc != L) atomicOr(&s_status, HPA_DEVICE_LEN_CLAMPED);
      p.ws.lens[b] = Lc;
      n = (Lc + kPageSize - 1) / kPageSize;
    }
    int total;
    const int before = block_exclusive_scan(n, s_warp, &total);
    if (b < p.B) p.ws.tile_start[b] = carry + before;
    carry += total;
  }
  if (tid == 0) p.ws.tile_start[p.B] = carry;
  __syncthreads();  // tile_start / lens visible block-wide

  const int32_t* ts = p.ws.tile_start;
  const long long T = carry;
  const long long U = T * p.Hkv;
  const int S = p.B * p.Hkv;
  const long long Pd = std::min<long long>(p.num_ctas, U);  // dynamic: active CTAs
  const int per = (p.kind == HPA_PLAN_DYNAMIC) ? 0 : p.grid / S;  // static: CTAs per segment

  // 2. per-CTA unit ranges and first-split indices
  for (int c = tid; c < p.grid; c += kPlanThreads) {
    long long ub, ue;
    int first = 0;
    if (p.kind == HPA_PLAN_DYNAMIC) {
      if (c < Pd) {
        ub = (long long)c * U / Pd;
        ue = (long long)(c + 1) * U / Pd;
        const int b = seq_of_unit(ts, p.B, p.Hkv, ub);
        const long long n = ts[b + 1] - ts[b];
        const long long g = (ub - (long long)ts[b] * p.Hkv) / n;
        const long long seg_start = (long long)ts[b] * p.Hkv + g * n;
        first = (int)(c - cta_of(seg_start, U, Pd));
      } else {
        ub = ue = U;
      }
    } else {
      const int s = c / per, i = c % per;
      const int b = s / p.Hkv, g = s % p.Hkv;
      const long long n = ts[b + 1] - ts[b];
      const long long C = (p.kind == HPA_PLAN_STATIC_NSPLIT) ? (n + per - 1) / per : p.chunk;
      const long long t0 = std::min<long long>((long long)i * C, n);
      const long long t1 = std::min<long long>((long long)(i + 1) * C, n);
      const long long seg_start = (long long)ts[b] * p.Hkv + (long long)g * n;
      ub = seg_start + t0;
      ue = seg_start + t1;
      first = t0 < t1 ? i : 0;
    }
    p.ws.cta_desc[c] = make_int4((int)ub, (int)ue, first, 0);
  }

  // 3. split counts, partial slot bases, zeroed arrival counters
  int pcarry = 0;
  for (int base = 0; base < S; base += kPlanThreads) {
    const int s = base + tid;
    int split = 0;
    if (s < S) {
      const int b = s / p.Hkv, g = s % p.Hkv;
      const long long n = ts[b + 1] - ts[b];
      if (n > 0) {
        if (p.kind == HPA_PLAN_DYNAMIC) {
          const long long seg_start = (long long)ts[b] * p.Hkv + (long long)g * n;
          split = (int)(cta_of(seg_start + n - 1, U, Pd) - cta_of(seg_start, U, Pd) + 1);
        } else {
          const long long C = (p.kind == HPA_PLAN_STATIC_NSPLIT) ? (n + per - 1) / per : p.chunk;
          split = (int)((n + C - 1) / C);
        }
      }
      p.ws.split_count[s] = split;
      p.ws.arrive[s] = 0;
    }
    int total;
    const int before = block_exclusive_scan(split > 1 ? split : 0, s_warp, &total);
    if (s < S) p.ws.part_base[s] = pcarry + before;
    pcarry += total;
  }

  __syncthreads();
  if (tid == 0) {
    int32_t* h = p.ws.header;
    h[kHdrStatus] = s_status;
    h[kHdrUnits] = (int32_t)U;
    h[kHdrGrid] = p.grid;
    h[kHdrKind] = p.kind;
    h[kHdrBatch] = p.B;
    h[kHdrKvHeads] = p.Hkv;
    h[kHdrGroup] = p.G;
    h[kHdrHeadDim] = p.D;
    h[kHdrTiles] = (int32_t)T;
    __threadfence();
    h[kHdrMagic] = kPlanMagic;
  }
  pdl_trigger();
}

}  // namespace
}  // namespace hpa

using namespace hpa;

extern "C" int hpa_plan_grid(hpa_plan_kind kind, int batch, int num_kv_heads, int num_ctas,
                             int param, int max_seq_len) {
  long long g = plan_grid_ll(kind, batch, num_kv_heads, num_ctas, param, max_seq_len, nullptr);
  if (g < 1 || g > (1LL << 30)) return -1;
  return (int)g;
}

extern "C" hpa_status hpa_decode_plan(const int32_t* seq_lens, int batch, int num_kv_heads,
                                      int num_q_heads, int head_dim, int pt_stride,
                                      hpa_plan_kind kind, int num_ctas, int param,
                                      int max_seq_len, void* workspace, size_t ws_bytes,
                                      int* grid_out, void* stream) {
  if (!seq_lens || !workspace || !grid_out) return HPA_ERR_INVALID_ARG;
  if (batch <= 0 || num_kv_heads <= 0 || num_q_heads <= 0 || pt_stride <= 0 || num_ctas <= 0 ||
      param < 0 || max_seq_len < 0)
    return HPA_ERR_INVALID_ARG;
  if (num_q_heads % num_kv_heads) return HPA_ERR_INVALID_ARG;
  if (kind != HPA_PLAN_DYNAMIC && kind != HPA_PLAN_STATIC_NSPLIT && kind != HPA_PLAN_STATIC_CHUNK)
    return HPA_ERR_INVALID_ARG;
  if ((long long)pt_stride * kPageSize > 0x7fffffffLL) return HPA_ERR_UNSUPPORTED;
  long long chunk = 0;
  const long long grid =
      plan_grid_ll(kind, batch, num_kv_heads, num_ctas, param, max_seq_len, &chunk);
  if (grid < 1 || grid > (1LL << 30)) return HPA_ERR_UNSUPPORTED;
  // Units are indexed with int32 in the plan: bound the worst case.
  if ((long long)batch * pt_stride * num_kv_heads > 0x7fffffffLL) return HPA_ERR_UNSUPPORTED;
  WsLayout L;
  if (!ws_layout(batch, num_kv_heads, num_q_heads, head_dim, (int)grid, &L))
    return HPA_ERR_INVALID_ARG;
  if (ws_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255)) return HPA_ERR_WORKSPACE;

  PlanParams p;
  p.seq_lens = seq_lens;
  p.B = batch;
  p.Hkv = num_kv_heads;
  p.G = num_q_heads / num_kv_heads;
  p.D = head_dim;
  p.capacity = pt_stride * kPageSize;
  p.kind = kind;
  p.num_ctas = num_ctas;
  p.grid = (int)grid;
  p.chunk = chunk;
  p.ws = ws_view(workspace, L);

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(kPlanThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, plan_kernel, p);
  if (e != cudaSuccess) {
    set_cuda_error(e, "hpa_decode_plan launch");
    return HPA_ERR_CUDA;
  }
  *grid_out = (int)grid;
  return HPA_OK;
}
