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
//
// The length-aware plan (HPA_PLAN_LENGTH_AWARE) is the same partition with
// its cut points moved to segment ends wherever they would leave a piece of
// fewer than m tiles (plan_geom.cuh, LaGeom): short sequences run whole in
// one range, long ones are spread in pieces of at least m tiles.
#include <algorithm>
#include <atomic>

#include "hpa_common.cuh"
#include "plan_geom.cuh"

namespace hpa {
namespace {

constexpr int kPlanThreads = 256;
constexpr int kPlanWarps = kPlanThreads / 32;
constexpr int kPlanMaxCtas = 64;  // each CTA repeats the length scan: keep the grid small

struct PlanParams {
  const int32_t* seq_lens;
  int B, Hkv, G, D, capacity;  // capacity = pt_stride * 64 tokens
  int kind, num_ctas, grid;
  long long chunk;             // STATIC_CHUNK: tiles per split; LENGTH_AWARE: smallest piece
  int tail_den, tail_chunks, tail_min;  // DYNAMIC / LENGTH_AWARE: the run-time tail's shape
  int unit_cost, end_cost;              // DYNAMIC / LENGTH_AWARE: cost weights of the primary cuts
  Ws ws;
};

__global__ void __launch_bounds__(kPlanThreads, 1) plan_kernel(PlanParams p) {
  // tile_start[0..B], then the non-empty mask and its prefix (SeqIdx), in
  // shared memory
  extern __shared__ int32_t ts[];
  const int nw = (p.B + 31) / 32;
  uint32_t* nzm = reinterpret_cast<uint32_t*>(ts + p.B + 1);
  int32_t* nzp = reinterpret_cast<int32_t*>(nzm + nw);
  __shared__ int s_warp[kPlanWarps], s_warp_nz[kPlanWarps];
  __shared__ int s_status;
  __shared__ double s_recip[4];
  // The previous step's run kernel may still be reading this workspace.
  pdl_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) s_status = 0;
  __syncthreads();

  // 1. clamped lengths -> tiles per sequence -> exclusive prefix sum, in
  //    shared memory.  Warp w scans its own contiguous slice (a multiple of
  //    32 entries) 32 entries at a time (coalesced loads, shuffle scans); the
  //    slices' totals are added after one barrier.  Alongside: which
  //    sequences have tiles, one mask word per 32, and the count before each.
  const int slice = ((p.B + kPlanWarps - 1) / kPlanWarps + 31) & ~31;
  const int lo = min(p.B, warp * slice), hi = min(p.B, lo + slice);
  int carry = 0, carry_nz = 0;
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
    const unsigned bal = __ballot_sync(0xffffffffu, n > 0);
    if (lane == 0) {
      nzm[i0 >> 5] = bal;
      nzp[i0 >> 5] = carry_nz;
    }
    carry_nz += __popc(bal);
  }
  if (lane == 0) {
    s_warp[warp] = carry;
    s_warp_nz[warp] = carry_nz;
  }
  __syncthreads();
  int off = 0, T = 0, off_nz = 0, T_nz = 0;
#pragma unroll
  for (int w = 0; w < kPlanWarps; ++w) {
    off += w < warp ? s_warp[w] : 0;
    T += s_warp[w];
    off_nz += w < warp ? s_warp_nz[w] : 0;
    T_nz += s_warp_nz[w];
  }
  if (off)
    for (int i = lo + lane; i < hi; i += 32) ts[i] += off;
  if (off_nz && lane == 0)
    for (int i0 = lo; i0 < hi; i0 += 32) nzp[i0 >> 5] += off_nz;
  if (tid == 0) {
    ts[p.B] = T;
    nzp[nw] = T_nz;
  }

  const long long U = (long long)T * p.Hkv;
  const int S = p.B * p.Hkv;
  const bool dyn = plan_is_dynamic(p.kind);
  const bool la = p.kind == HPA_PLAN_LENGTH_AWARE;
  const int per = dyn ? 0 : p.grid / S;  // static: CTAs per segment
  // (the tile offsets and the mask are complete: K(U1) reads them)
  __syncthreads();
  DynGeom dg;
  dg.init(U, p.num_ctas, p.tail_den, p.tail_chunks, p.tail_min, p.unit_cost, p.end_cost,
          SeqIdx{ts, nzm, nzp, p.B, p.Hkv}, lane);
  const LaGeom lg{&dg, ts, p.B, p.Hkv, la ? p.chunk : 1};
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
      int4 d0, d1;
      if (la) {
        la_range_desc(lg, c, &d0, &d1);
      } else if (dyn) {
        dyn_range_desc(dg, ts, p.B, p.Hkv, c, &d0, &d1);
      } else {
        const int s = (int)c / per, i = (int)c % per;
        const int b0 = s / p.Hkv, g0 = s % p.Hkv;
        const long long n = ts[b0 + 1] - ts[b0];
        const long long C = (p.kind == HPA_PLAN_STATIC_NSPLIT) ? (n + per - 1) / per : p.chunk;
        const long long c0 = std::min<long long>((long long)i * C, n);
        const long long c1 = std::min<long long>((long long)(i + 1) * C, n);
        const long long seg_start = (long long)ts[b0] * p.Hkv + (long long)g0 * n;
        d0 = make_int4((int)(seg_start + c0), (int)(seg_start + c1), b0, g0);
        d1 = make_int4((int)c0, (int)n, 0, 0);
      }
      p.ws.cta_desc[2 * c] = d0;
      p.ws.cta_desc[2 * c + 1] = d1;
    }
    if (c < S) {
      const int s = (int)c;
      if (la) {
        p.ws.seg_desc[s] = la_seg_desc(lg, s);
      } else if (dyn) {
        p.ws.seg_desc[s] = dyn_seg_desc(dg, ts, p.Hkv, s);
      } else {
        const int b = s / p.Hkv;
        const long long n = ts[b + 1] - ts[b];
        int nsplit = 0, slot0 = -1;
        if (n > 0) {
          const long long C = (p.kind == HPA_PLAN_STATIC_NSPLIT) ? (n + per - 1) / per : p.chunk;
          nsplit = (int)((n + C - 1) / C);
          if (nsplit > 1) slot0 = 2 * s * per;  // chunk 0 starts its segment
        }
        p.ws.seg_desc[s] = make_int2(slot0, nsplit);
      }
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
    h[kHdrDone] = 0;
    h[kHdrListCount] = 0;  // the in-kernel plan's merge list starts empty
    h[kHdrListCount + 1] = 0;
    h[kHdrParity] = 0;
    h[kHdrTailDen] = dyn ? p.tail_den : 0;
    h[kHdrTailChunks] = dyn ? p.tail_chunks : 0;
    h[kHdrTailMin] = dyn ? p.tail_min : 0;
    h[kHdrUnitCost] = dyn ? p.unit_cost : 0;
    h[kHdrEndCost] = dyn ? p.end_cost : 0;
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

namespace hpa {

// Shared memory of the plan kernel for `batch` sequences: tile offsets, the
// non-empty mask and its prefix.
static size_t plan_smem_bytes(int batch) {
  const size_t nw = (size_t(batch) + 31) / 32;
  return (size_t(batch) + 1) * 4 + nw * 4 + (nw + 1) * 4;
}

// hpa_decode_plan and hpa_decode_plan_shape: validation, parameters, launch.
static hpa_status plan_impl(const int32_t* seq_lens, int batch, int num_kv_heads,
                            int num_q_heads, int head_dim, int pt_stride, hpa_plan_kind kind,
                            int num_ctas, int param, int max_seq_len, int tail_den,
                            int tail_chunks, int tail_min, int unit_cost, int end_cost,
                            void* workspace, size_t ws_bytes, int* grid_out, void* stream) {
  if (!seq_lens || !workspace || !grid_out) return HPA_ERR_INVALID_ARG;
  if (batch <= 0 || num_kv_heads <= 0 || num_q_heads <= 0 || pt_stride <= 0 || num_ctas <= 0 ||
      param < 0 || max_seq_len < 0)
    return HPA_ERR_INVALID_ARG;
  if (num_q_heads % num_kv_heads) return HPA_ERR_INVALID_ARG;
  if (kind != HPA_PLAN_DYNAMIC && kind != HPA_PLAN_STATIC_NSPLIT && kind != HPA_PLAN_STATIC_CHUNK &&
      kind != HPA_PLAN_LENGTH_AWARE)
    return HPA_ERR_INVALID_ARG;
  if (tail_den < 0 || tail_den > (1 << 20) || tail_chunks < 1 || tail_chunks > HPA_TAIL_CHUNKS_MAX ||
      tail_min < 0 || tail_min > (1 << 20))
    return HPA_ERR_INVALID_ARG;
  if (unit_cost < 1 || unit_cost > HPA_COST_MAX || end_cost < 0 || end_cost > HPA_COST_MAX)
    return HPA_ERR_INVALID_ARG;
  if ((long long)pt_stride * kPageSize > 0x7fffffffLL) return HPA_ERR_UNSUPPORTED;
  if (batch > kMaxPlanBatch) return HPA_ERR_UNSUPPORTED;
  // the dynamic plan's range arithmetic keeps products below 2^50
  if (plan_is_dynamic(kind) && num_ctas > 65536) return HPA_ERR_UNSUPPORTED;
  if (kind == HPA_PLAN_LENGTH_AWARE && param > (1 << 20)) return HPA_ERR_UNSUPPORTED;
  long long chunk = 0;
  const long long grid =
      plan_grid_ll(kind, batch, num_kv_heads, num_ctas, param, max_seq_len, &chunk);
  if (kind == HPA_PLAN_LENGTH_AWARE) chunk = param > 0 ? param : kLaDefaultMinPiece;
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
  p.tail_den = tail_den;
  p.tail_chunks = tail_chunks;
  p.tail_min = tail_min;
  p.unit_cost = unit_cost;
  p.end_cost = end_cost;
  p.ws = ws_view(workspace, L);

  const size_t smem = plan_smem_bytes(batch);
  if (smem > 48 * 1024) {
    // tile offsets above 48 KiB of shared memory need the opt-in, once per device
    static std::atomic<uint64_t> ready_mask{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    const uint64_t bit = (e == cudaSuccess && dev < 64) ? (1ull << dev) : 0;
    if (!bit || !(ready_mask.load() & bit)) {
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)plan_smem_bytes(kMaxPlanBatch));
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

}  // namespace hpa

extern "C" hpa_status hpa_decode_plan(const int32_t* seq_lens, int batch, int num_kv_heads,
                                      int num_q_heads, int head_dim, int pt_stride,
                                      hpa_plan_kind kind, int num_ctas, int param,
                                      int max_seq_len, void* workspace, size_t ws_bytes,
                                      int* grid_out, void* stream) {
  return plan_impl(seq_lens, batch, num_kv_heads, num_q_heads, head_dim, pt_stride, kind,
                   num_ctas, param, max_seq_len, HPA_TAIL_DEN_DEFAULT, HPA_TAIL_CHUNKS_DEFAULT,
                   HPA_TAIL_MIN_DEFAULT, HPA_COST_UNIT_DEFAULT, HPA_COST_END_DEFAULT, workspace,
                   ws_bytes, grid_out, stream);
}

extern "C" hpa_status hpa_decode_plan_shape(const int32_t* seq_lens, int batch, int num_kv_heads,
                                            int num_q_heads, int head_dim, int pt_stride,
                                            hpa_plan_kind kind, int num_ctas, int param,
                                            int tail_den, int tail_chunks, int tail_min,
                                            int unit_cost, int end_cost, void* workspace,
                                            size_t ws_bytes, int* grid_out, void* stream) {
  if (!plan_is_dynamic(kind)) return HPA_ERR_INVALID_ARG;
  return plan_impl(seq_lens, batch, num_kv_heads, num_q_heads, head_dim, pt_stride, kind,
                   num_ctas, param, 0, tail_den, tail_chunks, tail_min, unit_cost, end_cost,
                   workspace, ws_bytes, grid_out, stream);
}
