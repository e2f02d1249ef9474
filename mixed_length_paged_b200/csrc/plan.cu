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
//
// The dynamic plan is a contiguous partition of the unit list into ranges:
// one primary range per persistent CTA over the first ~7/8 of the units, then
// small tail chunks that CTAs take at run time, in order, as they finish
// (bitbyai.com "vLLM x HPC-Ops", Attention Backend: the scheduler evaluates
// progress dynamically).  SMs do not all get the same share of HBM
// bandwidth, so equal static ranges would finish at different times; the
// tail evens that out.  The partition itself is fixed by the plan, so the
// split partials and their merge order -- and hence the result -- do not
// depend on which CTA ends up running a chunk.
#include <algorithm>
#include <atomic>

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
  constexpr int kWarps = kPlanThreads / 32;
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
    int w = lane < kWarps ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    s_warp[lane] = w;  // inclusive prefix of warp sums
  }
  __syncthreads();
  const int before = (warp > 0 ? s_warp[warp - 1] : 0) + x - v;
  *total = s_warp[kWarps - 1];
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

// floor(a / b) for 0 <= a < 2^50 and a fixed divisor 0 < b < 2^31: the fp64
// product with a precomputed reciprocal is within one of the quotient, and
// one integer check each way makes it exact.  (Much cheaper than a 64-bit
// integer division or an IEEE fp64 division per call.)
struct FloorDiv {
  long long b;
  double inv;
  __device__ void init(long long d, double reciprocal) {
    b = d;
    inv = reciprocal;
  }
  __device__ __forceinline__ long long operator()(long long a) const {
    long long q = (long long)((double)a * inv);
    if (q * b > a) --q;
    else if ((q + 1) * b <= a) ++q;
    return q;
  }
};

// Dynamic plan geometry.  P persistent CTAs; U units.  If U <= P each active
// CTA takes one unit.  Otherwise the first U1 = U - Ut units are spread over
// the P primary ranges and the last Ut = min(floor(U/8), U - P) units over M =
// min(4P, Ut) tail chunks, handed out at run time to whichever CTA is free.
// For n units spread over m ranges as [floor(cn/m), floor((c+1)n/m)), the
// range holding unit u is the largest c with floor(cn/m) <= u, i.e.
// floor(((u+1)m - 1) / n).
struct DynGeom {
  long long U, P, Pd, U1, Ut, M;
  FloorDiv by_Pd, by_M, by_U1, by_Ut;
  // r[0..3]: reciprocals of Pd, M, U1, Ut (0 for a zero divisor)
  __device__ void init_div(const double* r) {
    by_Pd.init(Pd, r[0]);
    by_M.init(M, r[1]);
    by_U1.init(U1, r[2]);
    by_Ut.init(Ut, r[3]);
  }
  __device__ long long range_of(long long u) const {
    return u < U1 ? by_U1((u + 1) * Pd - 1) : P + by_Ut((u - U1 + 1) * M - 1);
  }
};

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(PlanParams p) {
  extern __shared__ int32_t ts[];  // tile_start[0..B], in shared memory
  __shared__ int s_warp[32];
  __shared__ int s_status;
  __shared__ double s_recip[4];
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
    if (b < p.B) ts[b] = carry + before;
    carry += total;
  }
  if (tid == 0) ts[p.B] = carry;
  __syncthreads();
  for (int i = tid; i <= p.B; i += kPlanThreads) p.ws.tile_start[i] = ts[i];

  const long long T = carry;
  const long long U = T * p.Hkv;
  const int S = p.B * p.Hkv;
  const int per = (p.kind == HPA_PLAN_DYNAMIC) ? 0 : p.grid / S;  // static: CTAs per segment
  DynGeom dg;
  dg.U = U;
  dg.P = p.num_ctas;
  if (U <= dg.P) {
    dg.Pd = U; dg.U1 = U; dg.Ut = 0; dg.M = 0;
  } else {
    dg.Pd = dg.P;
    dg.Ut = std::min<long long>(U / kTailFractionDiv, U - dg.P);
    dg.U1 = U - dg.Ut;
    dg.M = std::min<long long>((long long)kTailChunksPerCta * dg.P, dg.Ut);
  }
  // the four reciprocals, computed once for the whole CTA
  if (tid < 4) {
    const long long d = tid == 0 ? dg.Pd : tid == 1 ? dg.M : tid == 2 ? dg.U1 : dg.Ut;
    s_recip[tid] = d > 0 ? 1.0 / (double)d : 0.0;
  }
  __syncthreads();
  dg.init_div(s_recip);
  const long long V = (p.kind == HPA_PLAN_DYNAMIC) ? dg.P + dg.M : p.grid;

  // 2. per-range unit ranges, first-split indices and start states
  for (int c = tid; c < V; c += kPlanThreads) {
    long long ub, ue;
    int first = 0, b0 = 0, g0 = 0, t0 = 0, n0 = 0;
    if (p.kind == HPA_PLAN_DYNAMIC) {
      if (c < dg.P) {
        if (c < dg.Pd) {
          ub = dg.by_Pd((long long)c * dg.U1);
          ue = dg.by_Pd((long long)(c + 1) * dg.U1);
        } else {
          ub = ue = U;
        }
      } else {
        const long long j = c - dg.P;
        ub = dg.U1 + dg.by_M(j * dg.Ut);
        ue = dg.U1 + dg.by_M((j + 1) * dg.Ut);
      }
      if (ub < ue) {
        b0 = seq_of_unit(ts, p.B, p.Hkv, ub);
        n0 = ts[b0 + 1] - ts[b0];
        const int rem = (int)(ub - (long long)ts[b0] * p.Hkv);  // < Hkv * n0 < 2^31
        g0 = rem / n0;
        t0 = rem - g0 * n0;
        const long long seg_start = (long long)ts[b0] * p.Hkv + (long long)g0 * n0;
        first = (int)(c - dg.range_of(seg_start));
      }
    } else {
      const int s = c / per, i = c % per;
      b0 = s / p.Hkv;
      g0 = s % p.Hkv;
      const long long n = ts[b0 + 1] - ts[b0];
      const long long C = (p.kind == HPA_PLAN_STATIC_NSPLIT) ? (n + per - 1) / per : p.chunk;
      const long long c0 = std::min<long long>((long long)i * C, n);
      const long long c1 = std::min<long long>((long long)(i + 1) * C, n);
      const long long seg_start = (long long)ts[b0] * p.Hkv + (long long)g0 * n;
      ub = seg_start + c0;
      ue = seg_start + c1;
      first = c0 < c1 ? i : 0;
      t0 = (int)c0;
      n0 = (int)n;
    }
    p.ws.cta_desc[2 * c] = make_int4((int)ub, (int)ue, first, b0);
    p.ws.cta_desc[2 * c + 1] = make_int4(g0, t0, n0, 0);
  }

  // 3. split counts and partial slot bases
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
          split = (int)(dg.range_of(seg_start + n - 1) - dg.range_of(seg_start) + 1);
        } else {
          const long long C = (p.kind == HPA_PLAN_STATIC_NSPLIT) ? (n + per - 1) / per : p.chunk;
          split = (int)((n + C - 1) / C);
        }
      }
      p.ws.split_count[s] = split;
    }
    int total;
    const int before = block_exclusive_scan(split > 1 ? split : 0, s_warp, &total);
    if (s < S) p.ws.part_base[s] = pcarry + before;
    pcarry += total;
  }

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
    h[kHdrRanges] = (int32_t)V;
    h[kHdrNext] = 0;
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
  if (batch > kMaxPlanBatch) return HPA_ERR_UNSUPPORTED;
  // the dynamic plan's range arithmetic keeps products below 2^50
  if (kind == HPA_PLAN_DYNAMIC && num_ctas > 65536) return HPA_ERR_UNSUPPORTED;
  long long chunk = 0;
  const long long grid =
      plan_grid_ll(kind, batch, num_kv_heads, num_ctas, param, max_seq_len, &chunk);
  if (grid < 1 || grid > (1LL << 30)) return HPA_ERR_UNSUPPORTED;
  // Units are indexed with int32 in the plan: bound the worst case.
  if ((long long)batch * pt_stride * num_kv_heads > 0x7fffffffLL) return HPA_ERR_UNSUPPORTED;
  WsLayout L;
  if (!ws_layout(kind, batch, num_kv_heads, num_q_heads, head_dim, (int)grid, &L))
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

  const size_t smem = (size_t(batch) + 1) * sizeof(int32_t);
  if (smem > 48 * 1024) {
    // tile offsets above 48 KiB of shared memory need the opt-in, once per device
    static std::atomic<uint64_t> ready_mask{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    const uint64_t bit = (e == cudaSuccess && dev < 64) ? (1ull << dev) : 0;
    if (!bit || !(ready_mask.load() & bit)) {
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)((size_t(kMaxPlanBatch) + 1) * sizeof(int32_t)));
      if (e != cudaSuccess) {
        set_cuda_error(e, "hpa_decode_plan smem attribute");
        return HPA_ERR_CUDA;
      }
      ready_mask.fetch_or(bit);
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(kPlanThreads);
  cfg.dynamicSmemBytes = smem;
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
