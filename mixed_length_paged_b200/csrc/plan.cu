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
// The plan is built on the device from the device-side lengths, so a decode
// step needs no host round trip.  Units are (sequence b, kv head g, tile t)
// in that order; segment s = b * Hkv + g.  Every CTA of the plan grid scans
// all lengths itself (a few hundred bytes for a typical batch) so that no CTA
// waits for another; the range and segment descriptors are then spread over
// the CTAs, each one a closed-form computation.
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

constexpr int kPlanThreads = 256;
constexpr int kPlanWarps = kPlanThreads / 32;
constexpr int kPlanMaxCtas = 64;  // each CTA repeats the length scan: keep the grid small

struct PlanParams {
  const int32_t* seq_lens;
  int B, Hkv, G, D, capacity;  // capacity = pt_stride * 64 tokens
  int kind, num_ctas, grid;
  long long chunk;             // STATIC_CHUNK: tiles per split
  Ws ws;
};

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
  __device__ void init(long long units, long long ctas) {
    U = units;
    P = ctas;
    if (U <= P) {
      Pd = U; U1 = U; Ut = 0; M = 0;
    } else {
      Pd = P;
      Ut = std::min<long long>(U / kTailFractionDiv, U - P);
      U1 = U - Ut;
      M = std::min<long long>((long long)kTailChunksPerCta * P, Ut);
    }
  }
  // the divisors whose reciprocals init_div takes, in order
  __device__ long long divisor(int i) const { return i == 0 ? Pd : i == 1 ? M : i == 2 ? U1 : Ut; }
  __device__ void init_div(const double* r) {
    by_Pd.init(Pd, r[0]);
    by_M.init(M, r[1]);
    by_U1.init(U1, r[2]);
    by_Ut.init(Ut, r[3]);
  }
  __device__ long long ranges() const { return P + M; }
  __device__ long long range_of(long long u) const {
    return u < U1 ? by_U1((u + 1) * Pd - 1) : P + by_Ut((u - U1 + 1) * M - 1);
  }
  __device__ void bounds(long long c, long long* ub, long long* ue) const {
    if (c < P) {
      if (c < Pd) {
        *ub = by_Pd(c * U1);
        *ue = by_Pd((c + 1) * U1);
      } else {
        *ub = *ue = U;
      }
    } else {
      const long long j = c - P;
      *ub = U1 + by_M(j * Ut);
      *ue = U1 + by_M((j + 1) * Ut);
    }
  }
};

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(PlanParams p) {
  extern __shared__ int32_t ts[];  // tile_start[0..B], in shared memory
  __shared__ int s_warp[kPlanWarps];
  __shared__ int s_status;
  __shared__ double s_recip[4];
  // The previous step's run kernel may still be reading this workspace.
  pdl_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) s_status = 0;
  __syncthreads();

  // 1. clamped lengths -> tiles per sequence -> exclusive prefix sum, in
  //    shared memory.  Warp w scans its own contiguous slice 32 entries at a
  //    time (coalesced loads, shuffle scans); the slices' totals are added
  //    after one barrier.
  const int slice = (p.B + kPlanWarps - 1) / kPlanWarps;
  const int lo = min(p.B, warp * slice), hi = min(p.B, lo + slice);
  int carry = 0;
  for (int i0 = lo; i0 < hi; i0 += 32) {
    const int i = i0 + lane;
    int n = 0;
    if (i < hi) {
      const int L = p.seq_lens[i];
      const int Lc = min(max(L, 0), p.capacity);
      if (Lc != L) atomicOr(&s_status, HPA_DEVICE_LEN_CLAMPED);
      n = (Lc + kPageSize - 1) / kPageSize;
    }
    int x = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (i < hi) ts[i] = carry + x - n;
    carry += __shfl_sync(0xffffffffu, x, 31);
  }
  if (lane == 0) s_warp[warp] = carry;
  __syncthreads();
  int off = 0, T = 0;
#pragma unroll
  for (int w = 0; w < kPlanWarps; ++w) {
    off += w < warp ? s_warp[w] : 0;
    T += s_warp[w];
  }
  if (off)
    for (int i = lo + lane; i < hi; i += 32) ts[i] += off;
  if (tid == 0) ts[p.B] = T;

  const long long U = (long long)T * p.Hkv;
  const int S = p.B * p.Hkv;
  const bool dyn = p.kind == HPA_PLAN_DYNAMIC;
  const int per = dyn ? 0 : p.grid / S;  // static: CTAs per segment
  DynGeom dg;
  dg.init(U, p.num_ctas);
  if (tid < 4) {
    const long long d = dg.divisor(tid);
    s_recip[tid] = d > 0 ? 1.0 / (double)d : 0.0;
  }
  __syncthreads();
  dg.init_div(s_recip);
  const long long V = dyn ? dg.ranges() : p.grid;
  const int stride = gridDim.x * kPlanThreads;
  const int first = blockIdx.x * kPlanThreads + tid;

  // lengths and tile offsets, written by all CTAs together
  for (int i = first; i <= p.B; i += stride) {
    p.ws.tile_start[i] = ts[i];
    if (i < p.B) p.ws.lens[i] = min(max(p.seq_lens[i], 0), p.capacity);
  }

  // 2. per range: its unit range and the state of its first unit; per
  //    segment: the ranges holding it and the slot of its first partial.
  //    (One loop, so that the two independent latency chains overlap.)
  const long long work = V > S ? V : S;
  for (long long c = first; c < work; c += stride) {
    if (c < V) {
      long long ub, ue;
      int b0 = 0, g0 = 0, t0 = 0, n0 = 0;
      if (dyn) {
        dg.bounds(c, &ub, &ue);
        if (ub < ue) {
          b0 = seq_of_unit(ts, p.B, p.Hkv, ub);
          n0 = ts[b0 + 1] - ts[b0];
          const int rem = (int)(ub - (long long)ts[b0] * p.Hkv);  // < Hkv * n0 < 2^31
          g0 = rem / n0;
          t0 = rem - g0 * n0;
        }
      } else {
        const int s = (int)c / per, i = (int)c % per;
        b0 = s / p.Hkv;
        g0 = s % p.Hkv;
        const long long n = ts[b0 + 1] - ts[b0];
        const long long C = (p.kind == HPA_PLAN_STATIC_NSPLIT) ? (n + per - 1) / per : p.chunk;
        const long long c0 = std::min<long long>((long long)i * C, n);
        const long long c1 = std::min<long long>((long long)(i + 1) * C, n);
        const long long seg_start = (long long)ts[b0] * p.Hkv + (long long)g0 * n;
        ub = seg_start + c0;
        ue = seg_start + c1;
        t0 = (int)c0;
        n0 = (int)n;
      }
      p.ws.cta_desc[2 * c] = make_int4((int)ub, (int)ue, b0, g0);
      p.ws.cta_desc[2 * c + 1] = make_int4(t0, n0, 0, 0);
    }
    if (c < S) {
      const int s = (int)c;
      const int b = s / p.Hkv, g = s - b * p.Hkv;
      const long long n = ts[b + 1] - ts[b];
      int nsplit = 0, slot0 = -1;
      if (n > 0) {
        if (dyn) {
          const long long seg_start = (long long)ts[b] * p.Hkv + (long long)g * n;
          const long long r0 = dg.range_of(seg_start);
          nsplit = (int)(dg.range_of(seg_start + n - 1) - r0 + 1);
          if (nsplit > 1) {
            long long ub, ue;
            dg.bounds(r0, &ub, &ue);
            slot0 = (int)(2 * r0 + (ub == seg_start ? 0 : 1));
          }
        } else {
          const long long C = (p.kind == HPA_PLAN_STATIC_NSPLIT) ? (n + per - 1) / per : p.chunk;
          nsplit = (int)((n + C - 1) / C);
          if (nsplit > 1) slot0 = 2 * s * per;  // chunk 0 starts its segment
        }
      }
      p.ws.seg_desc[s] = make_int2(slot0, nsplit);
    }
  }

  if (blockIdx.x == 0 && tid == 0) {
    int32_t* h = p.ws.header;
    h[kHdrStatus] = s_status;
    h[kHdrUnits] = (int32_t)U;
    h[kHdrGrid] = p.grid;
    h[kHdrKind] = p.kind;
    h[kHdrBatch] = p.B;
    h[kHdrKvHeads] = p.Hkv;
    h[kHdrGroup] = p.G;
    h[kHdrHeadDim] = p.D;
    h[kHdrTiles] = T;
    h[kHdrRanges] = (int32_t)V;
    h[kHdrNext] = 0;
    // (no fence before the magic word: the run kernel reads the plan only
    // after griddepcontrol.wait, i.e. after this whole grid has completed)
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
  const long long V = plan_ranges_ll(kind, (int)grid);
  const long long work = std::max<long long>(V, (long long)batch * num_kv_heads);
  const int ctas = (int)std::min<long long>(kPlanMaxCtas, (work + kPlanThreads - 1) / kPlanThreads);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(std::max(1, ctas));
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
