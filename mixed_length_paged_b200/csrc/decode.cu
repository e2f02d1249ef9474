// decode.cu -- persistent paged GQA decode attention (hpa_decode_run).
//
// The method (xiaodao.ai "HPC-Ops TPOT -48.8%", Attention section): persistent
// CTAs consume the planner's 64-token tile tasks; a (sequence, kv head) whose
// tiles span several CTAs is finished from per-split partials by a
// log-sum-exp merge.  The pages describe a Hopper design (TMA + WGMMA); this
// is written for sm_100a as follows.
//
// CTA = 4 consumer warps + 1 producer warp + 1 epilogue warp; one CTA per SM
// when the grid fits the SMs, two smaller co-resident CTAs per SM otherwise
// (twice the warps to hide each other's latencies).
//   producer: walks the CTA's unit range and resolves each unit's metadata
//     (page id, live tokens, first/last tile of its segment, partial slot,
//     FP8 scales) 32 units at a time, one per lane, so the global reads overlap.
//     For each unit it issues 2-D TMA loads of the K and V tiles of (page, kv
//     head) -- each a contiguous 64 x D block -- into a ring of shared-memory
//     stages with 128-byte swizzle (bank-conflict-free fragment loads) and an
//     L2 evict-first hint; for the first tile of a segment it also bulk-copies
//     the segment's query rows.  The metadata rides along in the stage.
//   consumers: warp w owns tokens [16w, 16w+16) of every tile and keeps its own
//     online-softmax state (m, l, acc) for the tile's query rows:
//       S^T[16 tok x 8 rows] = K_w[16 x D] . Q^T        (mma m16n8k16, fp32 acc)
//       online softmax in base 2 (logits pre-scaled by scale * log2 e)
//       O^T[D x 8 rows]    += V_w^T[D x 16] . P^T      (P^T built in registers
//                                                      with movmatrix)
//     The query rows of a kv head (G heads, times T tokens for multi-token
//     decode) sit on the MMA N dimension, 8 per n-tile, padded.  With 9..16
//     rows (two n-tiles) warp w instead owns n-tile w / 2 and tokens
//     [32 (w % 2), +32), which keeps the registers of the one-n-tile kernel.
//     At a segment end each warp deposits its state in a double-buffered
//     shared-memory slot and carries on.
//   epilogue: combines the states of the warps holding each row of a
//     deposited segment; a segment held whole by the CTA is written directly,
//     otherwise the CTA stores an (acc, m, l) partial.  This keeps the
//     consumers streaming through segment boundaries.
// Each stage has two full barriers: one for its small copies (query rows;
// the new token's raw K/V rows under the fused prologue) and one for the K/V
// tiles, so work on the former overlaps the tiles' load.
// A second, small kernel (chained by programmatic dependent launch) merges
// the partials of every split segment in range order, one warp per (segment,
// row), all partials loaded in parallel.  (Merging inside the persistent
// kernel puts a single CTA's dependent L2 reads on the critical path: the
// splits of a long sequence all finish together at the end of the step.)
//
// Fused prologue (hpa_decode_run_prologue): the consumers normalise and
// rotate the raw query rows of each piece in shared memory; the warp whose
// tokens hold the new token's slot patches its K/V rows into the landed tile
// and stores them to the cache.  Multi-token decode (hpa_decode_run_multi):
// row n = token n / G of T; each column masks the positions past its token.
//
// FP8 (e4m3) caches: K/V codes are converted in registers with
// cvt.rn.f16x2.e4m3x2 (exact) and the products run as f16 MMAs; the
// per-(page, kv head) K scale folds into that tile's logits and the V scale
// into its probabilities.  To keep the e4m3 -> f16 conversion on whole
// registers, the D index inside each 16-wide MMA step is permuted (the same
// permutation on both operands, so the dot products are unchanged) and the
// output rows are un-permuted when deposited.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>

#include <cuda_bf16.h>

#include "hpa_common.cuh"
#include "plan_geom.cuh"
#include "prologue_math.cuh"

namespace hpa {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kProducerWarp = kConsumerWarps;
constexpr int kEpilogueWarp = kConsumerWarps + 1;
constexpr int kThreads = (kConsumerWarps + 2) * 32;
constexpr int kSmemLimit = 227 * 1024;   // per CTA
constexpr int kSmemPerSm = 228 * 1024;
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s bound on any barrier wait
constexpr int kDepBufsDefault = 2;              // deposit slots between consumers and epilogue
constexpr int kMaxQTokens = 16;          // query tokens per sequence (multi-token decode)

template <int D, int NT, bool FP8, int CPS, bool PRO, bool FP>
struct Cfg {
  static constexpr int kElt = FP8 ? 1 : 2;
  static constexpr int kRowBytes = D * kElt;           // one token row of one head
  static constexpr int kBoxes = kRowBytes / 128;       // 128-byte-wide TMA boxes per tile
  static constexpr int kBoxBytes = kPageSize * 128;    // 8 KiB
  static constexpr int kTileBytes = kPageSize * kRowBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;   // K tile + V tile
  static constexpr int kHeads = 8 * NT;                // MMA N (padded group)
  static constexpr int kQBytes = kHeads * D * 2;       // a segment's bf16 query rows
  // fused prologue: the new token's raw K and V rows ride behind the q rows
  static constexpr int kRawBytes = PRO ? 2 * D * 2 : 0;
  static constexpr int kSlotBytes = kQBytes + kRawBytes; // per-stage q (+ raw rows) slot
  static constexpr int kAccStride = D + 4;             // floats; keeps deposits off one bank
  // Warp roles.  One n-tile (8 rows): warp w owns tokens [16w, 16w + 16) of
  // every tile and all 8 rows.  Two n-tiles (9..16 rows): warp w owns n-tile
  // w / 2 and tokens [32 (w % 2), + 32), as two 16-token blocks -- the same
  // MMA work with the registers of the one-n-tile kernel, so two CTAs still
  // fit an SM.  Four n-tiles (17..32 rows): warp w owns n-tile w and all 64
  // tokens, as four 16-token blocks.  The 32 query rows of a stage take 8 KiB
  // more shared memory, so at two CTAs per SM this kernel keeps one deposit
  // buffer (two stages fit then); at one CTA per SM it keeps two.
  static constexpr bool kSplit = NT >= 2;
  static constexpr int kWarpsPerTile = kSplit ? kConsumerWarps / NT : kConsumerWarps;
  static constexpr int kWarpTiles = kSplit ? 1 : NT;   // n-tiles per warp
  static constexpr int kBlocks = kSplit ? NT : 1;      // 16-token blocks per warp
  static constexpr int kWarpRows = 8 * kWarpTiles;     // rows each warp deposits
  static constexpr int kRowWarps = kSplit ? kWarpsPerTile : kConsumerWarps;  // warps holding a row
  static_assert(NT == 1 || NT == 2 || NT == 4, "one, two or four n-tiles");
  // one deposit: acc[warp][row of the warp][D + 4] floats, then (m, l)[warp][row]
  static constexpr int kDepAccFloats = kConsumerWarps * kWarpRows * kAccStride;
  static constexpr int kDepBytes = kDepAccFloats * 4 + kConsumerWarps * kWarpRows * 8;
  // deposit slots between consumers and epilogue: one for the four-n-tile
  // kernel at two CTAs per SM (its 8 KiB of query rows per stage leave room
  // for two stages only then), else two
  static constexpr int kDepBufs = (NT == 4 && CPS == 2) ? 1 : kDepBufsDefault;
  static constexpr int kMisc = 2048;                   // barriers, stage info, flags
  // in-kernel plan: tile offsets of all sequences, the non-empty mask and
  // its prefix (SeqIdx), and the scan's per-warp non-empty counts
  static constexpr int kTsWords = (kMaxFusedBatch + 1) + kMaxFusedBatch / 32 +
                                  (kMaxFusedBatch / 32 + 1) + kThreads / 32;
  static constexpr int kTsBytes = FP ? (kTsWords * 4 + 15) / 16 * 16 : 0;
  // CPS CTAs share one SM's 228 KiB (1 KiB of it reserved per CTA)
  static constexpr int kBudget = CPS == 1 ? kSmemLimit : (kSmemPerSm / CPS - 1024);
  static constexpr int kStagesFit =
      (kBudget - 1024 - kDepBufs * kDepBytes - kMisc - kTsBytes) / (kStageBytes + kSlotBytes);
  static constexpr int kStages = kStagesFit < 8 ? kStagesFit : 8;
  static constexpr int kSmemBytes =
      1024 + kStages * (kStageBytes + kSlotBytes) + kDepBufs * kDepBytes + kMisc + kTsBytes;
  static constexpr int kKSteps = D / 16;               // QK MMA k-steps
  static constexpr int kMTiles = D / 16;               // PV MMA m-tiles
  static constexpr int kVec = D / 32;                  // output floats per epilogue lane
  static_assert(kRowBytes % 128 == 0, "tile rows must be whole 128-byte boxes");
  static_assert(kStages >= 2, "not enough shared memory for a pipeline");
  static_assert(kDepBytes % 16 == 0, "deposit slots must stay 16-byte aligned");
};

struct RunParams {
  const uint16_t* q;        // bf16 bits [B][Hq][D] (raw, pre-norm rows under the fused prologue)
  const float* k_scale;     // [pages][Hkv] (FP8)
  const float* v_scale;
  const int32_t* page_table;
  int pt_stride, num_pages;
  void* out;
  float* lse;               // optional [B][T][Hq] log-sum-exp of each output row (natural log)
  int B, Hq, Hkv, G;
  int T, GT;                // query tokens per sequence; rows per kv head = G * T
  const int32_t* seq_lens;  // in-kernel plan: the step's lengths (else the plan's)
  int capacity;             // in-kernel plan: pt_stride * 64 tokens
  int tail_den, tail_chunks, tail_min;  // in-kernel plan: the run-time tail's shape
  int unit_cost, end_cost;              // in-kernel plan: cost weights of the primary cuts
  float scale_log2;         // softmax_scale * log2(e)
  Ws ws;
  int grid, kind;
  int slots;                // 2 * V partial slots in the workspace
  // fused prologue only: raw new-token K/V rows, weights, caches to write
  const __nv_bfloat16* k_raw;  // [B][Hkv][D]
  const __nv_bfloat16* v_raw;
  const float* q_gamma;        // [D]
  const float* k_gamma;
  float eps;
  double log2_theta;
  __nv_bfloat16* k_cache_w;    // the K/V caches the TMA maps read
  __nv_bfloat16* v_cache_w;
  __nv_bfloat16* q_out;        // optional copy of the normalised, rotated q
};

// What the producer resolved for the unit held in one stage.
constexpr int kFirst = 1;   // first tile of its segment in this range
constexpr int kLast = 2;    // last tile of its segment in this range
constexpr int kEnd = 4;     // no unit: the producer has no more work
constexpr int kNewTok = 8;  // fused prologue: the tile that receives the new token
constexpr int kSegStart = 16;  // tile 0 of its segment
struct alignas(16) StageInfo {
  int32_t b, g, valid, flags;   // sequence, kv head, live tokens in the tile, k* flags
  int32_t slot, pos, row, pad;   // partial slot of the segment's piece (-1: whole
                                 // segment); fused prologue: new token's position,
                                 // first cache row of the tile
  float k_scale, v_scale, pad2, pad3;
};

// Segment handed from the consumers to the epilogue warp.
struct alignas(16) DepDesc {
  int32_t b, g, slot, stop, pad0, pad1, pad2, pad3;
};

// 2^x on the SFU (ex2.approx, flush-to-zero): relative error ~2^-22, and
// 2^-inf = +0, which the masked logits rely on.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Bounded barrier wait; on timeout (or an earlier abort) records the failure
// and returns false.  Never spins without bound.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         int32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  if (*abort_flag) return false;
  const uint64_t t0 = globaltimer();
  for (uint32_t i = 0; i < (1u << 28); ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 63) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > kWaitNs) break;
    }
  }
  *abort_flag = 1;
  atomicOr(status, HPA_DEVICE_TIMEOUT);
  return false;
}

// Walk over (b, g, t) units in global order; n = tiles of sequence b.
struct Walk {
  int b, g, t, n;
  __device__ void next(const int32_t* ts, int Hkv) {
    if (++t < n) return;
    t = 0;
    if (++g < Hkv) return;
    g = 0;
    do {
      ++b;
      n = ts[b + 1] - ts[b];
    } while (n == 0);
  }
};

// Natural-log log-sum-exp of a row from its softmax state: M the running
// max and lam = sum 2^(s_j - M) over the scaled logits s_j = scale * log2(e)
// * q.k_j, so log sum_j e^(scale q.k_j) = (M + log2 lam) * ln 2.  A row that
// saw no token (lam = 0) has -inf.
__device__ __forceinline__ float lse_of(float M, float lam) {
  return lam > 0.f ? (M + log2f(lam)) * 0.69314718055994531f : -INFINITY;
}

template <bool OUT_F32>
__device__ __forceinline__ void store_out(void* out, long long i, float v) {
  if constexpr (OUT_F32) reinterpret_cast<float*>(out)[i] = v;
  else reinterpret_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16_rn(v);
}

// Stores kVec consecutive outputs starting at element i (i a multiple of kVec).
template <bool OUT_F32, int kVec>
__device__ __forceinline__ void store_out_vec(void* out, long long i, const float (&v)[kVec]) {
  if constexpr (OUT_F32) {
    if constexpr (kVec == 4) *reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + i) = make_float4(v[0], v[1], v[2], v[3]);
    else *reinterpret_cast<float2*>(reinterpret_cast<float*>(out) + i) = make_float2(v[0], v[1]);
  } else {
    if constexpr (kVec == 4) {
      uint2 w;
      w.x = pack_bf16(v[0], v[1]);
      w.y = pack_bf16(v[2], v[3]);
      *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(out) + i) = w;
    } else {
      *reinterpret_cast<uint32_t*>(reinterpret_cast<__nv_bfloat16*>(out) + i) = pack_bf16(v[0], v[1]);
    }
  }
}

template <int D, int NT, bool FP8, bool OUT_F32, int CPS, bool PRO, bool FP>
__global__ void __launch_bounds__(kThreads, CPS)
    decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const RunParams p) {
  using C = Cfg<D, NT, FP8, CPS, PRO, FP>;
  static_assert(!(PRO && FP8), "the fused prologue writes bf16 caches");
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned in the shared window (the 128-byte swizzle needs it),
  // derived by offsetting smem_raw so that every pointer below stays a
  // shared-memory pointer to the compiler
  const uint32_t smem_raw_s = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((smem_raw_s + 1023u) & ~1023u) - smem_raw_s);
  uint8_t* stages = smem;
  uint8_t* qslots = smem + C::kStages * C::kStageBytes;
  uint8_t* deps = qslots + C::kStages * C::kSlotBytes;  // C::kDepBufs deposit slots
  uint8_t* misc = deps + C::kDepBufs * C::kDepBytes;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(misc);
  uint64_t* empty_bar = full_bar + C::kStages;
  uint64_t* dep_full = empty_bar + C::kStages;
  uint64_t* dep_empty = dep_full + C::kDepBufs;
  uint64_t* q_full = dep_empty + C::kDepBufs;  // a stage's small copies (q rows, raw rows) landed
  // StageInfo / DepDesc are read and written as 16-byte vectors: the first
  // 16-byte boundary after the barriers (misc is 16-byte aligned; an offset
  // from it keeps the pointer in the shared space for the compiler)
  StageInfo* info =
      reinterpret_cast<StageInfo*>(misc + ((C::kStages * 24 + C::kDepBufs * 16 + 15) & ~15));
  DepDesc* dep_desc = reinterpret_cast<DepDesc*>(info + C::kStages);
  volatile int* s_flags = reinterpret_cast<volatile int*>(dep_desc + C::kDepBufs);
  volatile int* s_abort = s_flags;
  volatile int* s_plan_ok = s_flags + 1;
  uint64_t* q_ready = reinterpret_cast<uint64_t*>(const_cast<int*>(s_flags) + 2);  // fused prologue: q rows done
  // fused prologue: RMSNorm weights, in the upper half of the misc area
  float* s_qgamma = reinterpret_cast<float*>(misc + C::kMisc / 2);
  float* s_kgamma = s_qgamma + D;
  static_assert(C::kMisc / 2 >= 2 * D * 4, "misc area too small for the weights");
  static_assert(C::kStages * 24 + C::kDepBufs * 16 + 8 + C::kStages * sizeof(StageInfo) +
                        C::kDepBufs * sizeof(DepDesc) + 16 + 32 <= C::kMisc / 2,
                "misc area too small");
  // in-kernel plan: tile offsets, non-empty mask and prefix, per-warp
  // non-empty counts (after the misc area), and per-warp tile sums of the
  // scan (behind q_ready)
  int32_t* s_ts = reinterpret_cast<int32_t*>(misc + C::kMisc);
  uint32_t* s_nzm = reinterpret_cast<uint32_t*>(s_ts + kMaxFusedBatch + 1);
  int32_t* s_nzp = reinterpret_cast<int32_t*>(s_nzm + kMaxFusedBatch / 32);
  int* s_wnz = s_nzp + kMaxFusedBatch / 32 + 1;
  int* s_wsum = const_cast<int*>(s_flags) + 4;
  volatile int* s_parity = s_flags + 10;  // in-kernel plan: step parity (after the warp sums)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&q_full[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), kConsumerWarps);
    }
    for (int d = 0; d < C::kDepBufs; ++d) {
      mbar_init(smem_u32(&dep_full[d]), kConsumerWarps);
      mbar_init(smem_u32(&dep_empty[d]), 1);
    }
    mbar_init(smem_u32(q_ready), kConsumerWarps * 32);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  // Everything below reads what the plan (and possibly the prologue) wrote.
  pdl_wait();
  const uint64_t t_cta0 = globaltimer();  // this CTA's start, for the trace region
  if constexpr (FP) {
    // In-kernel plan (hpa_decode_step): every CTA turns the step's lengths
    // into tile offsets and the non-empty mask in shared memory, as the plan
    // kernel does -- warp w scans a contiguous slice (a multiple of 32) 32
    // lengths at a time -- and then derives its own ranges from the same
    // closed forms.
    constexpr int kW = kThreads / 32;
    const int slice = ((p.B + kW - 1) / kW + 31) & ~31;
    const int lo = min(p.B, warp * slice), hi = min(p.B, lo + slice);
    int carry = 0, carry_nz = 0;
    bool clamped = false;
    for (int i0 = lo; i0 < hi; i0 += 32) {
      const int i = i0 + lane;
      int n = 0;
      if (i < hi) {
        const int L = p.seq_lens[i];
        const int Lc = min(max(L, 0), p.capacity);
        clamped |= Lc != L;
        n = (Lc + kPageSize - 1) / kPageSize;
      }
      int x = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (i < hi) s_ts[i] = carry + x - n;
      carry += __shfl_sync(0xffffffffu, x, 31);
      if constexpr (FP8) {
        const unsigned bal = __ballot_sync(0xffffffffu, n > 0);
        if (lane == 0) {
          s_nzm[i0 >> 5] = bal;
          s_nzp[i0 >> 5] = carry_nz;
        }
        carry_nz += __popc(bal);
      }
    }
    if (lane == 0) {
      s_wsum[warp] = carry;
      s_wnz[warp] = carry_nz;
    }
    if (blockIdx.x == 0 && __any_sync(0xffffffffu, clamped) && lane == 0)
      atomicOr(&p.ws.header[kHdrStatus], HPA_DEVICE_LEN_CLAMPED);
    __syncthreads();
    int off = 0, T = 0, off_nz = 0, T_nz = 0;
#pragma unroll
    for (int w = 0; w < kW; ++w) {
      off += w < warp ? s_wsum[w] : 0;
      T += s_wsum[w];
      off_nz += w < warp ? s_wnz[w] : 0;
      T_nz += s_wnz[w];
    }
    if (off)
      for (int i = lo + lane; i < hi; i += 32) s_ts[i] += off;
    if (off_nz && lane == 0)
      for (int i0 = lo; i0 < hi; i0 += 32) s_nzp[i0 >> 5] += off_nz;
    if (threadIdx.x == 0) {
      s_ts[p.B] = T;
      s_nzp[(p.B + 31) >> 5] = T_nz;
      *s_plan_ok = 1;
      *s_parity = __ldcg(&p.ws.header[kHdrParity]) & 1;  // this step's merge-list count
    }
  } else if (threadIdx.x == 0) {
    const int32_t* h = p.ws.header;
    const bool ok = h[kHdrMagic] == kPlanMagic && h[kHdrGrid] == p.grid &&
                    h[kHdrGrid] == (int)gridDim.x && h[kHdrBatch] == p.B &&
                    h[kHdrKvHeads] == p.Hkv && h[kHdrGroup] == p.GT && h[kHdrHeadDim] == D &&
                    h[kHdrKind] == p.kind && h[kHdrRanges] >= p.grid &&
                    h[kHdrRanges] <= plan_ranges_ll(p.kind, p.grid);
    *s_plan_ok = ok;
    if (!ok) atomicOr(&p.ws.header[kHdrStatus], HPA_DEVICE_BAD_PLAN);
  }
  if constexpr (PRO) {
    for (int i = threadIdx.x; i < D; i += kThreads) {
      s_qgamma[i] = p.q_gamma[i];
      s_kgamma[i] = p.k_gamma[i];
    }
  }
  __syncthreads();
  if (!*s_plan_ok) return;
  pdl_trigger();

  int32_t* status = &p.ws.header[kHdrStatus];
  const int32_t* ts = FP ? s_ts : p.ws.tile_start;
  // clamped length of sequence b
  auto len_of = [&](int b) -> int {
    if constexpr (FP) return min(max(p.seq_lens[b], 0), p.capacity);
    else return p.ws.lens[b];
  };
  // the dynamic plan's geometry (in-kernel plan only)
  DynGeom dg{};
  if constexpr (FP) {
    if (warp >= kConsumerWarps) {
      // (cost weights only for e4m3 caches: with end cost 0 the cost code
      // drops out of the bf16 kernels)
      dg.init((long long)ts[p.B] * p.Hkv, gridDim.x, p.tail_den, p.tail_chunks, p.tail_min,
              FP8 ? p.unit_cost : 1, FP8 ? p.end_cost : 0, SeqIdx{ts, s_nzm, s_nzp, p.B, p.Hkv},
              lane);
      double rc[4];
      dyn_reciprocals(dg, rc);
      dg.init_div(rc);
    }
  }

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    const uint64_t policy = l2_policy_evict_first();
    const int qrow_bytes = p.G * D * 2;  // one query token's rows of a kv head group
    const int qbytes = p.T * qrow_bytes;
    const int U = FP ? (int)dg.U : p.ws.header[kHdrUnits];
    const int V = FP ? (int)dg.ranges() : p.ws.header[kHdrRanges];
    const bool dyn = plan_is_dynamic(p.kind);  // tail chunks taken at run time
    int it = 0;
    // This CTA's primary range first; under the dynamic plan it then takes
    // tail chunks, reserving the next one (and reading its descriptor) while
    // it streams the current one.
    int v = blockIdx.x;
    int4 d0, d1;
    if constexpr (FP) {
      dyn_range_desc(dg, ts, p.B, p.Hkv, v, &d0, &d1, lane);
    } else {
      d0 = p.ws.cta_desc[2 * v];
      d1 = p.ws.cta_desc[2 * v + 1];
    }
    while (true) {
      int vn = V;
      int4 n0 = make_int4(0, 0, 0, 0), n1 = n0;
      if (dyn) {
        if (lane == 0) vn = p.grid + atomicAdd(&p.ws.header[kHdrNext], 1);
        vn = __shfl_sync(0xffffffffu, vn, 0);
        if (vn < V) {
          if constexpr (FP) {
            dyn_range_desc(dg, ts, p.B, p.Hkv, vn, &n0, &n1);
          } else {
            n0 = p.ws.cta_desc[2 * vn];
            n1 = p.ws.cta_desc[2 * vn + 1];
          }
        }
      }
      const int ub = max(0, d0.x), ue = min(d0.y, U);
      Walk wk{d0.z, d0.w, d1.x, d1.y};
      if (ub < ue && (wk.b < 0 || wk.b >= p.B || wk.n <= 0 || wk.n != ts[wk.b + 1] - ts[wk.b] ||
                      wk.g < 0 || wk.g >= p.Hkv || wk.t < 0 || wk.t >= wk.n)) {
        if (lane == 0) atomicOr(status, HPA_DEVICE_BAD_PLAN);
      } else {
        for (int u0 = ub; u0 < ue; u0 += 32) {
          Walk w2 = wk;
          for (int k = 0; k < lane && u0 + k + 1 < ue; ++k) w2.next(ts, p.Hkv);
          const int u = u0 + lane;
          int row = 0, valid = 0, flags = 0, slot = -1, bad = 0, pos = 0;
          float ks = 1.f, vs = 1.f;
          if (u < ue) {
            const int page = __ldg(p.page_table + (long long)w2.b * p.pt_stride + w2.t);
            const int L = len_of(w2.b);
            // tokens from the tile's start to the sequence end, capped where no
            // query row's limit can reach (multi-token rows see up to T - 1 fewer)
            valid = min(kPageSize + kMaxQTokens - 1, L - w2.t * kPageSize);
            flags = ((w2.t == 0 || u == ub) ? kFirst : 0) | ((w2.t == w2.n - 1 || u == ue - 1) ? kLast : 0) |
                    (w2.t == 0 ? kSegStart : 0) | ((PRO && w2.t == w2.n - 1) ? kNewTok : 0);
            pos = L - 1;  // the new token's position (post-append length - 1)
            if (flags & kLast) {
              // The piece of this segment in range v is whole if the segment
              // starts inside the range and ends here.  Otherwise it is a
              // partial: slot 2v if the segment is the range's first, else
              // 2v + 1 (it is then the range's last).
              const int useg = u - w2.t;  // unit of the segment's tile 0
              if (useg < ub || w2.t != w2.n - 1) slot = 2 * v + (useg > ub ? 1 : 0);
            }
            if (page < 0 || page >= p.num_pages) {
              bad = 1;
            } else {
              row = (page * p.Hkv + w2.g) * kPageSize;
              if constexpr (FP8) {
                ks = __ldg(p.k_scale + page * p.Hkv + w2.g);
                vs = __ldg(p.v_scale + page * p.Hkv + w2.g);
              }
            }
          }
          // small fields travel packed: valid (7 bits) | flags (5) | bad (1) | g (<< 13)
          const int packed = valid | (flags << 7) | (bad << 12) | (w2.g << 13);
          const int cnt = min(32, ue - u0);
          for (int k = 0; k < cnt; ++k) {
            const int rk = __shfl_sync(0xffffffffu, row, k);
            const int pk = __shfl_sync(0xffffffffu, packed, k);
            StageInfo si;
            si.b = __shfl_sync(0xffffffffu, w2.b, k);
            si.g = pk >> 13;
            si.valid = pk & 127;
            si.flags = (pk >> 7) & 31;
            const int bk = (pk >> 12) & 1;
            si.slot = -1;
            if (si.flags & kLast)  // warp-uniform: pk is the same in every lane
              si.slot = __shfl_sync(0xffffffffu, slot, k);
            si.pos = PRO ? __shfl_sync(0xffffffffu, pos, k) : 0;
            si.pad = 0;
            si.k_scale = si.v_scale = 1.f;
            if constexpr (FP8) {
              si.k_scale = __shfl_sync(0xffffffffu, ks, k);
              si.v_scale = __shfl_sync(0xffffffffu, vs, k);
            }
            si.pad2 = si.pad3 = 0.f;
            si.row = rk;
            if (bk) si.flags &= ~kNewTok;  // no tile, no new row
            if (lane == 0) {
              const int s = it % C::kStages;
              const uint32_t par = ((it / C::kStages) & 1) ^ 1;
              const uint32_t fb = smem_u32(&full_bar[s]), qb = smem_u32(&q_full[s]);
              if (wait_bar(smem_u32(&empty_bar[s]), par, s_abort, status) && !bk) {
                info[s] = si;
                const bool first = si.flags & kFirst;
                const bool newtok = PRO && (si.flags & kNewTok);
                // The small copies complete on q_full, so that the consumers
                // can prepare the query (and the new K row) while the K/V
                // tiles, which complete on full_bar, are still in flight.
                mbar_arrive_expect_tx(qb, (first ? qbytes : 0) + (newtok ? 4 * D : 0));
                if (first)  // rows n = i * G + h: query token i, head h of the group
                  for (int i = 0; i < p.T; ++i)
                    bulk_load(smem_u32(qslots + s * C::kSlotBytes) + i * qrow_bytes,
                              p.q + (((long long)si.b * p.T + i) * p.Hq + (long long)si.g * p.G) * D,
                              qrow_bytes, qb);
                if (newtok) {
                  // the new token's raw K and V rows, for the consumers to
                  // patch into this tile
                  const long long src = ((long long)si.b * p.Hkv + si.g) * D;
                  const uint32_t raw = smem_u32(qslots + s * C::kSlotBytes + C::kQBytes);
                  bulk_load(raw, p.k_raw + src, 2 * D, qb);
                  bulk_load(raw + 2 * D, p.v_raw + src, 2 * D, qb);
                }
                mbar_arrive_expect_tx(fb, C::kStageBytes);
                const uint32_t kdst = smem_u32(stages + s * C::kStageBytes);
                const uint32_t vdst = kdst + C::kTileBytes;
    #pragma unroll
                for (int bx = 0; bx < C::kBoxes; ++bx) {
                  const int x = bx * (128 / C::kElt);
                  tma_load_2d(kdst + bx * C::kBoxBytes, &tm_k, x, rk, fb, policy);
                  tma_load_2d(vdst + bx * C::kBoxBytes, &tm_v, x, rk, fb, policy);
                }
              } else {
                info[s] = si;
                if (bk) atomicOr(status, HPA_DEVICE_BAD_PAGE);
                mbar_arrive(qb);  // release the consumers without data (result void)
                mbar_arrive(fb);
              }
            }
            __syncwarp();
            ++it;
          }
          for (int k = 0; k < cnt; ++k)
            if (u0 + k + 1 < ue) wk.next(ts, p.Hkv);
        }
      }
      if (!dyn || vn >= V || *s_abort) break;
      v = vn;
      d0 = n0;
      d1 = n1;
    }
    // end of work: a stage without data whose info says so
    if (lane == 0) {
      const int s = it % C::kStages;
      const uint32_t par = ((it / C::kStages) & 1) ^ 1;
      if (wait_bar(smem_u32(&empty_bar[s]), par, s_abort, status)) {
        StageInfo si = {};
        si.flags = kEnd;
        info[s] = si;
        mbar_arrive(smem_u32(&q_full[s]));
        mbar_arrive(smem_u32(&full_bar[s]));
      }
    }
    __syncwarp();
    ++it;
    if (lane == 0) {
      // trace: start, end of the producer's work, units streamed
      unsigned long long* tr = p.ws.trace + 4ull * blockIdx.x;
      tr[0] = t_cta0;
      tr[1] = globaltimer();
      tr[3] = (unsigned long long)(it - 1);
    }
    // zero output rows of empty sequences (a softmax over no tokens), for
    // every query token
    for (int b = blockIdx.x; b < p.B; b += gridDim.x) {
      if (len_of(b) != 0) continue;
      const long long n = (long long)p.T * p.Hq * D;
      for (long long i = lane; i < n; i += 32) store_out<OUT_F32>(p.out, (long long)b * n + i, 0.f);
      if (p.lse)
        for (int i = lane; i < p.T * p.Hq; i += 32) p.lse[(long long)b * p.T * p.Hq + i] = -INFINITY;
    }
    // After an abort, make sure no copy is still landing in shared memory.
    if (lane == 0 && *s_abort) {
      const int first = max(0, it - C::kStages);
      for (int j = first; j < it; ++j) {
        const int s = j % C::kStages;
        const uint32_t fb = smem_u32(&full_bar[s]), qb = smem_u32(&q_full[s]);
        const uint64_t t0 = globaltimer();
        while (!(mbar_try_wait(fb, (j / C::kStages) & 1) && mbar_try_wait(qb, (j / C::kStages) & 1)) &&
               globaltimer() - t0 < kWaitNs) {
        }
      }
    }
    if (dyn) {
      // The last CTA out resets the tail-chunk counter for the next step, so
      // that a step whose plan is made in the kernel (hpa_decode_step) finds
      // it at 0 whatever ran before on this workspace.  Every CTA gets here
      // once (aborted ones too), after its last ticket, so the counter is no
      // longer in use then.
      if (lane == 0) {
        __threadfence();
        if (atomicAdd(&p.ws.header[kHdrDone], 1) == (int)gridDim.x - 1) {
          atomicExch(&p.ws.header[kHdrNext], 0);
          atomicExch(&p.ws.header[kHdrDone], 0);
          if constexpr (FP) {
            // The merge list: empty the previous step's count (its merge has
            // finished: this kernel started after it) and flip the parity,
            // so the next step appends there.  Every CTA read the parity
            // before its producer started, so none reads the new value.
            const int e = *s_parity;
            atomicExch(&p.ws.header[kHdrListCount + (e ^ 1)], 0);
            atomicExch(&p.ws.header[kHdrParity], e ^ 1);
          }
        }
      }
    }
    return;
  }

  if (warp == kEpilogueWarp) {
    // ------------------------------------------------------------ epilogue
    const int GT = p.GT;  // rows per kv head: query token i, head h at row i * G + h
    constexpr int V = C::kVec;
    if constexpr (FP) {
      // In-kernel plan: the segment descriptors the merge reads, shared out
      // over the CTAs, and (CTA 0) the plan fields of the header.
      const int S = p.B * p.Hkv;
      // Each split segment (more than one piece) also goes on the merge
      // list: one atomic per warp batch reserves its entries.
      for (int sg0 = blockIdx.x * 32; sg0 < S; sg0 += gridDim.x * 32) {
        const int sg = sg0 + lane;
        const int2 sd = sg < S ? dyn_seg_desc(dg, ts, p.Hkv, sg) : make_int2(-1, 0);
        if (sg < S) p.ws.seg_desc[sg] = sd;
        const unsigned split = __ballot_sync(0xffffffffu, sd.y > 1);
        if (split) {
          int base = 0;
          if (lane == 0) base = atomicAdd(&p.ws.header[kHdrListCount + *s_parity], __popc(split));
          base = __shfl_sync(0xffffffffu, base, 0);
          const int at = base + __popc(split & ((1u << lane) - 1u));
          // (with its descriptor, so that the merge reads one word less in
          // its chain of dependent loads; a stale count is flagged by the merge)
          if (sd.y > 1 && at >= 0 && at < S) p.ws.mlist[at] = make_int4(sg, sd.x, sd.y, 0);
        }
      }
      if (blockIdx.x == 0 && lane == 0) {
        int32_t* h = p.ws.header;
        h[kHdrUnits] = (int32_t)dg.U;
        h[kHdrGrid] = p.grid;
        h[kHdrKind] = HPA_PLAN_DYNAMIC;
        h[kHdrBatch] = p.B;
        h[kHdrKvHeads] = p.Hkv;
        h[kHdrGroup] = p.GT;
        h[kHdrHeadDim] = D;
        h[kHdrTiles] = ts[p.B];
        h[kHdrRanges] = (int32_t)dg.ranges();
        h[kHdrTailDen] = p.tail_den;
        h[kHdrTailChunks] = p.tail_chunks;
        h[kHdrTailMin] = p.tail_min;
        h[kHdrUnitCost] = FP8 ? p.unit_cost : 1;
        h[kHdrEndCost] = FP8 ? p.end_cost : 0;
        h[kHdrMagic] = kPlanMagic;
      }
    }
    for (int k = 0;; ++k) {
      const int db = k % C::kDepBufs;
      if (!wait_bar(smem_u32(&dep_full[db]), (k / C::kDepBufs) & 1, s_abort, status)) break;
      DepDesc dd = dep_desc[db];
      if (dd.stop) break;
      // Never trust a deposit as an index without checking it.
      if (dd.b < 0 || dd.b >= p.B || dd.g < 0 || dd.g >= p.Hkv || dd.slot >= p.slots) {
        if (lane == 0) atomicOr(status, HPA_DEVICE_BAD_PLAN);
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&dep_empty[db]));
        continue;
      }
      const float* dacc = reinterpret_cast<const float*>(deps + db * C::kDepBytes);
      const float2* dml = reinterpret_cast<const float2*>(dacc + C::kDepAccFloats);
      const int d = lane * V;
      // combine the states of the warps that hold each row, two rows at a
      // time: both rows' deposits are read before either is combined, so
      // their shared-memory latencies overlap
      constexpr int R = C::kRowWarps;
      auto load_row = [&](int h, float2 (&ml)[R], float (&a)[R][V]) {
        const int w0 = C::kSplit ? R * (h >> 3) : 0;  // first warp holding row h
        const int lr = C::kSplit ? (h & 7) : h;       // its row inside those warps
#pragma unroll
        for (int k = 0; k < R; ++k) {
          ml[k] = dml[(w0 + k) * C::kWarpRows + lr];
          const float* src = dacc + ((w0 + k) * C::kWarpRows + lr) * C::kAccStride + d;
          if constexpr (V == 4) {
            const float4 x = *reinterpret_cast<const float4*>(src);
            a[k][0] = x.x; a[k][1] = x.y; a[k][2] = x.z; a[k][3] = x.w;
          } else {
            const float2 x = *reinterpret_cast<const float2*>(src);
            a[k][0] = x.x; a[k][1] = x.y;
          }
        }
      };
      auto finish_row = [&](int h, const float2 (&ml)[R], const float (&a)[R][V]) {
        float M = -INFINITY;
#pragma unroll
        for (int k = 0; k < R; ++k) M = fmaxf(M, ml[k].x);
        float lam = 0.f, o[V];
#pragma unroll
        for (int v = 0; v < V; ++v) o[v] = 0.f;
#pragma unroll
        for (int k = 0; k < R; ++k) {
          // a warp that saw no token of the piece holds m = -inf, acc = 0
          const float sc = (ml[k].x == -INFINITY) ? 0.f : fast_exp2(ml[k].x - M);
          lam += ml[k].y * sc;
#pragma unroll
          for (int v = 0; v < V; ++v) o[v] += a[k][v] * sc;
        }
        if (dd.slot < 0) {
          // a row that sees no token (a query ahead of the sequence) is 0
          const float inv = lam > 0.f ? 1.f / lam : 0.f;
#pragma unroll
          for (int v = 0; v < V; ++v) o[v] *= inv;
          const int qi = h / p.G, hh = h - qi * p.G;
          const long long orow = ((long long)dd.b * p.T + qi) * p.Hq + (long long)dd.g * p.G + hh;
          store_out_vec<OUT_F32, V>(p.out, orow * D + d, o);
          if (p.lse && lane == 0) p.lse[orow] = lse_of(M, lam);
        } else {
          float* dst = p.ws.part_acc + ((long long)dd.slot * GT + h) * D + d;
          if constexpr (V == 4) *reinterpret_cast<float4*>(dst) = make_float4(o[0], o[1], o[2], o[3]);
          else *reinterpret_cast<float2*>(dst) = make_float2(o[0], o[1]);
          if (lane == 0) p.ws.part_ml[(long long)dd.slot * GT + h] = make_float2(M, lam);
        }
      };
      int h = 0;
      for (; h + 1 < GT; h += 2) {
        float2 ml0[R], ml1[R];
        float a0[R][V], a1[R][V];
        load_row(h, ml0, a0);
        load_row(h + 1, ml1, a1);
        finish_row(h, ml0, a0);
        finish_row(h + 1, ml1, a1);
      }
      if (h < GT) {
        float2 ml0[R];
        float a0[R][V];
        load_row(h, ml0, a0);
        finish_row(h, ml0, a0);
      }
      // the deposit slot is free again
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&dep_empty[db]));
    }
    if (lane == 0) p.ws.trace[4ull * blockIdx.x + 2] = globaltimer();  // trace: epilogue done
    return;
  }

  // -------------------------------------------------------------- consumers
  constexpr int W = C::kWarpTiles, MB = C::kBlocks;
  const int r = lane >> 2, c = lane & 3;          // MMA fragment coordinates
  const int lm = lane >> 3, lr = lane & 7;        // ldmatrix address lane roles
  const int nt0 = C::kSplit ? warp / C::kWarpsPerTile : 0;  // this warp's first n-tile
  const int tok0 = C::kSplit ? (kPageSize / C::kWarpsPerTile) * (warp % C::kWarpsPerTile)
                             : 16 * warp;                   // its first token
  // ldmatrix row (token) for the QK A operand and the PV A operand
  const int k_tok = tok0 + (lm & 1) * 8 + lr;
  const int k_chk = lm >> 1;
  const int v_tok = FP8 ? tok0 + (lm & 1) * 8 + lr : tok0 + (lm >> 1) * 8 + lr;
  const int v_chk = FP8 ? (lm >> 1) : (lm & 1);
  // Byte offsets (inside a tile) of this lane's ldmatrix rows for chunk 2j +
  // chk, j = 0..3, under the 128-byte swizzle; chunk 2j + 8 + chk adds one
  // box, and the next 16-token block adds 16 rows of 128 bytes (the swizzle
  // pattern repeats every 8 rows).
  constexpr uint32_t kBlockBytes = 16 * 128;
  uint32_t koff[4], voff[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    koff[j] = k_tok * 128 + ((((2 * j + k_chk) & 7) ^ (k_tok & 7)) << 4);
    voff[j] = v_tok * 128 + ((((2 * j + v_chk) & 7) ^ (v_tok & 7)) << 4);
  }

  uint32_t qf[W][C::kKSteps][2];
  float acc[W][C::kMTiles][4];
  float m_run[W][2], l_run[W][2];
  int nseg = 0;  // segments deposited so far
  // Multi-token decode: column n of the MMA N dimension is query token n / G;
  // it sees T - 1 - n / G tokens fewer than the last one (padding columns
  // past G * T see what the last one sees).
  int kshift[W][2];
#pragma unroll
  for (int nt = 0; nt < W; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) kshift[nt][e] = max(0, p.T - 1 - ((nt0 + nt) * 8 + 2 * c + e) / p.G);
  int nq = 0;    // fused prologue: q_ready phases completed
  RopeLane<D> rope;  // fused prologue: cos/sin at the current piece's new-token position

  // Hand this warp's state of a finished segment to the epilogue warp.
  auto deposit = [&](const StageInfo* inf) {
    const int db = nseg % C::kDepBufs;
    wait_bar(smem_u32(&dep_empty[db]), ((nseg / C::kDepBufs) & 1) ^ 1, s_abort, status);
    if (inf) {
#pragma unroll
      for (int nt = 0; nt < W; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float v = l_run[nt][e];
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          l_run[nt][e] = v;
        }
      float* dacc = reinterpret_cast<float*>(deps + db * C::kDepBytes);
      float2* dml = reinterpret_cast<float2*>(dacc + C::kDepAccFloats);
      float* my_acc = dacc + warp * C::kWarpRows * C::kAccStride;
#pragma unroll
      for (int nt = 0; nt < W; ++nt) {
        const int h0 = nt * 8 + 2 * c;  // row inside this warp's rows
#pragma unroll
        for (int i = 0; i < C::kMTiles; ++i) {
          const int dr0 = FP8 ? 16 * i + 2 * r : 16 * i + r;
          const int dr1 = FP8 ? dr0 + 1 : dr0 + 8;
          my_acc[h0 * C::kAccStride + dr0] = acc[nt][i][0];
          my_acc[(h0 + 1) * C::kAccStride + dr0] = acc[nt][i][1];
          my_acc[h0 * C::kAccStride + dr1] = acc[nt][i][2];
          my_acc[(h0 + 1) * C::kAccStride + dr1] = acc[nt][i][3];
        }
        if (r == 0) {
          dml[warp * C::kWarpRows + h0] = make_float2(m_run[nt][0], l_run[nt][0]);
          dml[warp * C::kWarpRows + h0 + 1] = make_float2(m_run[nt][1], l_run[nt][1]);
        }
      }
    }
    if (warp == 0 && lane == 0) {
      DepDesc dd;
      dd.b = inf ? inf->b : -1;
      dd.g = inf ? inf->g : 0;
      dd.slot = inf ? inf->slot : -1;
      dd.stop = inf ? 0 : 1;
      dd.pad0 = dd.pad1 = dd.pad2 = dd.pad3 = 0;
      dep_desc[db] = dd;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&dep_full[db]));
    ++nseg;
  };

  // V fragments (MMA A operand of O^T += V^T P^T) of 16-token block mb.
  auto load_v = [&](uint32_t vt, int mb, uint32_t (&va)[C::kMTiles][4]) {
    const uint32_t vb = vt + mb * kBlockBytes;
    if constexpr (!FP8) {
#pragma unroll
      for (int i = 0; i < C::kMTiles; ++i)
        ldsm_x4_t(vb + voff[i & 3] + (i >> 2) * C::kBoxBytes, va[i][0], va[i][1], va[i][2], va[i][3]);
    } else {
#pragma unroll
      for (int ip = 0; ip < C::kMTiles / 2; ++ip) {
        uint32_t r0, r1, r2, r3;
        ldsm_x4_t(vb + voff[ip], r0, r1, r2, r3);
        // r0/r1: tokens [0,8)/[8,16) of chunk 2ip; r2/r3: same for chunk 2ip+1.
        // Each holds bytes {V(t,d), V(t,d+1), V(t+1,d), V(t+1,d+1)}.
        // one byte permutation per register: {b0, b2} in the low half, {b1, b3}
        // in the high half
        const uint32_t t0 = __byte_perm(r0, 0, 0x3120), t1 = __byte_perm(r1, 0, 0x3120);
        const uint32_t t2 = __byte_perm(r2, 0, 0x3120), t3 = __byte_perm(r3, 0, 0x3120);
        va[2 * ip][0] = e4m3x2_to_f16x2((uint16_t)(t0 & 0xffffu));
        va[2 * ip][1] = e4m3x2_to_f16x2((uint16_t)(t0 >> 16));
        va[2 * ip][2] = e4m3x2_to_f16x2((uint16_t)(t1 & 0xffffu));
        va[2 * ip][3] = e4m3x2_to_f16x2((uint16_t)(t1 >> 16));
        va[2 * ip + 1][0] = e4m3x2_to_f16x2((uint16_t)(t2 & 0xffffu));
        va[2 * ip + 1][1] = e4m3x2_to_f16x2((uint16_t)(t2 >> 16));
        va[2 * ip + 1][2] = e4m3x2_to_f16x2((uint16_t)(t3 & 0xffffu));
        va[2 * ip + 1][3] = e4m3x2_to_f16x2((uint16_t)(t3 >> 16));
      }
    }
  };

  for (int it = 0;; ++it) {
    const int s = it % C::kStages;
    const uint32_t par = (it / C::kStages) & 1;
    if (!wait_bar(smem_u32(&q_full[s]), par, s_abort, status)) break;
    const StageInfo inf = info[s];
    if (inf.flags & kEnd) break;
    const uint32_t kt = smem_u32(stages + s * C::kStageBytes);
    const uint32_t vt = kt + C::kTileBytes;

    if (inf.flags & kFirst) {
      if constexpr (PRO) {
        // RMSNorm + RoPE of the G raw query rows, in place in the stage's q
        // slot: consumer warp w takes rows w, w + 4, ...; the piece holding
        // the segment's tile 0 also writes them out.  Every lane arrives on
        // q_ready after its stores, and all wait for all.
        __nv_bfloat16* qrows = reinterpret_cast<__nv_bfloat16*>(qslots + s * C::kSlotBytes);
        rope.init(inf.pos, lane, p.log2_theta);  // kept for this piece's new K row
        for (int h = warp; h < p.G; h += kConsumerWarps) {
          __nv_bfloat16* qo = (p.q_out && (inf.flags & kSegStart))
                                  ? p.q_out + ((long long)inf.b * p.Hq + (long long)inf.g * p.G + h) * D
                                  : nullptr;
          norm_rope_row<D>(qrows + h * D, qrows + h * D, qo, s_qgamma, p.eps, rope, lane);
        }
        // the slot is refilled by a bulk copy once the stage is released
        fence_proxy_async_shared();
        mbar_arrive(smem_u32(q_ready));
        if (!wait_bar(smem_u32(q_ready), nq & 1, s_abort, status)) break;
        ++nq;
      }
      // query fragments (MMA B operand) of this warp's rows
      const uint16_t* qs = reinterpret_cast<const uint16_t*>(qslots + s * C::kSlotBytes);
#pragma unroll
      for (int nt = 0; nt < W; ++nt) {
        const int hh = (nt0 + nt) * 8 + r;
        const bool hv = hh < p.GT;
        const uint16_t* qrow = qs + hh * D;
#pragma unroll
        for (int ks = 0; ks < C::kKSteps; ++ks) {
          if constexpr (!FP8) {
            qf[nt][ks][0] = hv ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * c) : 0u;
            qf[nt][ks][1] = hv ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 8 + 2 * c) : 0u;
          } else {
            // permuted k index: step ks covers d = 16 ks + 4c + {0,1} and {2,3}
            const uint2 raw = hv ? *reinterpret_cast<const uint2*>(qrow + 16 * ks + 4 * c) : make_uint2(0, 0);
            const float x0 = __uint_as_float(raw.x << 16), x1 = __uint_as_float(raw.x & 0xffff0000u);
            const float x2 = __uint_as_float(raw.y << 16), x3 = __uint_as_float(raw.y & 0xffff0000u);
            qf[nt][ks][0] = pack_f16(x0, x1);
            qf[nt][ks][1] = pack_f16(x2, x3);
          }
        }
#pragma unroll
        for (int i = 0; i < C::kMTiles; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[nt][i][j] = 0.f;
        m_run[nt][0] = m_run[nt][1] = -INFINITY;
        l_run[nt][0] = l_run[nt][1] = 0.f;
      }
    }

    // Fused prologue: if the new token's row lies in this warp's tokens, form
    // its K row (RMSNorm + RoPE of the raw row; the piece's cos/sin are
    // already in `rope`) while the tiles are still in flight.  (With two
    // n-tiles, the two warps on the slot's tokens both patch it, with the
    // same bits.)
    const int ptok = inf.pos & (kPageSize - 1);
    const bool patch = PRO && (inf.flags & kNewTok) && ptok >= tok0 && ptok < tok0 + 16 * MB;
    __nv_bfloat16 klo[D / 64], khi[D / 64];
    if constexpr (PRO) {
      if (patch)
        norm_rope_vals<D>(reinterpret_cast<const __nv_bfloat16*>(qslots + s * C::kSlotBytes + C::kQBytes),
                          s_kgamma, p.eps, rope, lane, klo, khi);
    }

    if (!wait_bar(smem_u32(&full_bar[s]), par, s_abort, status)) break;

    if constexpr (PRO) {
      if (patch) {
        // patch the new K and V rows into the landed tiles (128-byte
        // swizzle) and write them to their cache slot
        const int tr = ptok;
        const uint4* vraw = reinterpret_cast<const uint4*>(qslots + s * C::kSlotBytes + C::kQBytes + 2 * D);
        uint8_t* ktile = stages + s * C::kStageBytes;
        uint8_t* vtile = ktile + C::kTileBytes;
        __nv_bfloat16* kdst = p.k_cache_w + ((long long)inf.row + tr) * D;
        uint4* vdst = reinterpret_cast<uint4*>(p.v_cache_w + ((long long)inf.row + tr) * D);
        // byte offset of 16-byte chunk j (of D * 2 / 16) of row tr inside a tile
        auto chunk_off = [&](int j) {
          return (j >> 3) * C::kBoxBytes + tr * 128 + (((j & 7) ^ (tr & 7)) << 4);
        };
#pragma unroll
        for (int j = 0; j < D / 64; ++j) {
          const int i = lane + 32 * j, i2 = i + D / 2;
          *reinterpret_cast<__nv_bfloat16*>(ktile + chunk_off(i >> 3) + (i & 7) * 2) = klo[j];
          *reinterpret_cast<__nv_bfloat16*>(ktile + chunk_off(i2 >> 3) + (i2 & 7) * 2) = khi[j];
          kdst[i] = klo[j];
          kdst[i2] = khi[j];
        }
        if (lane < D / 8) {
          const uint4 v = vraw[lane];
          *reinterpret_cast<uint4*>(vtile + chunk_off(lane)) = v;
          vdst[lane] = v;
        }
        // the stage is refilled by TMA once released
        fence_proxy_async_shared();
        __syncwarp();
      }
    }

    // ---- S^T = K_w . Q^T per 16-token block, four independent accumulation
    // chains (k-step mod 4)
    constexpr int kChains = 4;
    float sacc[MB][W][4];
#pragma unroll
    for (int mb = 0; mb < MB; ++mb) {
      const uint32_t kb = kt + mb * kBlockBytes;
      float sch[kChains][W][4];
#pragma unroll
      for (int q = 0; q < kChains; ++q)
#pragma unroll
        for (int nt = 0; nt < W; ++nt)
#pragma unroll
          for (int j = 0; j < 4; ++j) sch[q][nt][j] = 0.f;
      if constexpr (!FP8) {
#pragma unroll
        for (int ks = 0; ks < C::kKSteps; ++ks) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(kb + koff[ks & 3] + (ks >> 2) * C::kBoxBytes, a0, a1, a2, a3);
#pragma unroll
          for (int nt = 0; nt < W; ++nt)
            mma_bf16(sch[ks % kChains][nt], a0, a1, a2, a3, qf[nt][ks][0], qf[nt][ks][1]);
        }
      } else {
#pragma unroll
        for (int kp = 0; kp < C::kKSteps / 2; ++kp) {
          uint32_t r0, r1, r2, r3;
          ldsm_x4(kb + koff[kp], r0, r1, r2, r3);
          const uint32_t a[2][4] = {
              {e4m3x2_to_f16x2(r0 & 0xffff), e4m3x2_to_f16x2(r1 & 0xffff), e4m3x2_to_f16x2(r0 >> 16),
               e4m3x2_to_f16x2(r1 >> 16)},
              {e4m3x2_to_f16x2(r2 & 0xffff), e4m3x2_to_f16x2(r3 & 0xffff), e4m3x2_to_f16x2(r2 >> 16),
               e4m3x2_to_f16x2(r3 >> 16)}};
#pragma unroll
          for (int nt = 0; nt < W; ++nt) {
            mma_f16(sch[(2 * kp) % kChains][nt], a[0][0], a[0][1], a[0][2], a[0][3],
                    qf[nt][2 * kp][0], qf[nt][2 * kp][1]);
            mma_f16(sch[(2 * kp + 1) % kChains][nt], a[1][0], a[1][1], a[1][2], a[1][3],
                    qf[nt][2 * kp + 1][0], qf[nt][2 * kp + 1][1]);
          }
        }
      }
#pragma unroll
      for (int nt = 0; nt < W; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j)
          sacc[mb][nt][j] = (sch[0][nt][j] + sch[1][nt][j]) + (sch[2][nt][j] + sch[3][nt][j]);
    }

    // V fragments of the first block now, so their shared-memory latency
    // overlaps the softmax
    uint32_t va[C::kMTiles][4];
    load_v(vt, 0, va);
    if constexpr (MB == 1) {
      // all shared-memory reads of this stage are issued: hand it back
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty_bar[s]));
    }

    // ---- online softmax (base 2) over this warp's MB blocks
    // tokens from this warp's first token to the sequence end; query row n
    // (token n / G of the T new ones) sees kshift[n] of them fewer
    const int valid = inf.valid - tok0;
    const float mul = p.scale_log2 * inf.k_scale;
    uint32_t pb[MB][W][2];
    float alpha[W][2];
#pragma unroll
    for (int nt = 0; nt < W; ++nt) {
      float sv[MB][4];
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int mb = 0; mb < MB; ++mb) {
        sv[mb][0] = sacc[mb][nt][0] * mul;
        sv[mb][1] = sacc[mb][nt][1] * mul;
        sv[mb][2] = sacc[mb][nt][2] * mul;
        sv[mb][3] = sacc[mb][nt][3] * mul;
        const int vb = valid - 16 * mb;  // tokens from this block's start
        if (vb - (p.T - 1) < 16) {       // warp-uniform: some logit of the block is masked
          const int lim0 = vb - kshift[nt][0], lim1 = vb - kshift[nt][1];
          if (r >= lim0) sv[mb][0] = -INFINITY;
          if (r >= lim1) sv[mb][1] = -INFINITY;
          if (r + 8 >= lim0) sv[mb][2] = -INFINITY;
          if (r + 8 >= lim1) sv[mb][3] = -INFINITY;
        }
        mx0 = fmaxf(mx0, fmaxf(sv[mb][0], sv[mb][2]));
        mx1 = fmaxf(mx1, fmaxf(sv[mb][1], sv[mb][3]));
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 4));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 4));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 8));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 8));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 16));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 16));
      const float mn0 = fmaxf(m_run[nt][0], mx0), mn1 = fmaxf(m_run[nt][1], mx1);
      const float base0 = (mn0 == -INFINITY) ? 0.f : mn0;
      const float base1 = (mn1 == -INFINITY) ? 0.f : mn1;
      const float al0 = fast_exp2(m_run[nt][0] - base0), al1 = fast_exp2(m_run[nt][1] - base1);
      float l0 = l_run[nt][0] * al0, l1 = l_run[nt][1] * al1;
#pragma unroll
      for (int mb = 0; mb < MB; ++mb) {
        const float p0 = fast_exp2(sv[mb][0] - base0), p2 = fast_exp2(sv[mb][2] - base0);
        const float p1 = fast_exp2(sv[mb][1] - base1), p3 = fast_exp2(sv[mb][3] - base1);
        l0 += p0 + p2;
        l1 += p1 + p3;
        if constexpr (!FP8) {
          pb[mb][nt][0] = movm_t(pack_bf16(p0, p1));
          pb[mb][nt][1] = movm_t(pack_bf16(p2, p3));
        } else {
          const float vsc = inf.v_scale;
          pb[mb][nt][0] = movm_t(pack_f16(p0 * vsc, p1 * vsc));
          pb[mb][nt][1] = movm_t(pack_f16(p2 * vsc, p3 * vsc));
        }
      }
      l_run[nt][0] = l0;
      l_run[nt][1] = l1;
      m_run[nt][0] = mn0;
      m_run[nt][1] = mn1;
      alpha[nt][0] = al0;
      alpha[nt][1] = al1;
    }
    // Rescale the accumulators only if some running max moved (once the
    // maxima settle, almost no tile needs it).
    bool moved = false;
#pragma unroll
    for (int nt = 0; nt < W; ++nt) moved |= (alpha[nt][0] != 1.f) | (alpha[nt][1] != 1.f);
    if (__any_sync(0xffffffffu, moved)) {
#pragma unroll
      for (int nt = 0; nt < W; ++nt)
#pragma unroll
        for (int i = 0; i < C::kMTiles; ++i) {
          acc[nt][i][0] *= alpha[nt][0];
          acc[nt][i][1] *= alpha[nt][1];
          acc[nt][i][2] *= alpha[nt][0];
          acc[nt][i][3] *= alpha[nt][1];
        }
    }

    // ---- O^T += V_w^T . P^T per block   (V rows past the length are zeroed
    // in registers: their probabilities are 0 but the slot may hold NaN/Inf
    // garbage)
#pragma unroll
    for (int mb = 0; mb < MB; ++mb) {
      if (mb > 0) {
        load_v(vt, mb, va);
        if (mb == MB - 1) {
          // all shared-memory reads of this stage are issued: hand it back
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&empty_bar[s]));
        }
      }
      const int vb = valid - 16 * mb;
      if (vb < 16) {  // warp-uniform: some V row of the block is past the end
        const uint32_t m_lo = (2 * c < vb ? 0x0000ffffu : 0u) | (2 * c + 1 < vb ? 0xffff0000u : 0u);
        const uint32_t m_hi = (2 * c + 8 < vb ? 0x0000ffffu : 0u) | (2 * c + 9 < vb ? 0xffff0000u : 0u);
#pragma unroll
        for (int i = 0; i < C::kMTiles; ++i) {
          va[i][0] &= m_lo;
          va[i][1] &= m_lo;
          va[i][2] &= m_hi;
          va[i][3] &= m_hi;
        }
      }
#pragma unroll
      for (int i = 0; i < C::kMTiles; ++i)
#pragma unroll
        for (int nt = 0; nt < W; ++nt) {
          if constexpr (!FP8)
            mma_bf16(acc[nt][i], va[i][0], va[i][1], va[i][2], va[i][3], pb[mb][nt][0], pb[mb][nt][1]);
          else
            mma_f16(acc[nt][i], va[i][0], va[i][1], va[i][2], va[i][3], pb[mb][nt][0], pb[mb][nt][1]);
        }
    }

    if (inf.flags & kLast) deposit(&inf);
  }
  deposit(nullptr);  // tells the epilogue warp that this CTA is done
}


// ---------------------------------------------------------------------------
// Split merge: for every segment with more than one piece, the log-sum-exp
// combination of its partials in range order,
//   M = max_i m_i,  Lambda = sum_i l_i 2^(m_i - M),  o = sum_i acc_i 2^(m_i - M) / Lambda
// (m in log2 units).  One warp per (segment, head), D / 32 output elements
// per lane.  The slots follow from the segment descriptor, so after that one
// read the warp issues the (m, l) of up to 32 pieces (one per lane) and its
// share of their partial rows together: two L2 round trips in all for a
// segment of at most kMergeBatch pieces.  Lane j forms piece j's weight; the
// weights reach the other lanes by shuffle.
// ---------------------------------------------------------------------------
constexpr int kMergeWarps = 4;

// L2-only loads kept in program order (a batch is issued before any of its
// values is used).
__device__ __forceinline__ float2 ld_cg2(const float2* p) {
  float2 v;
  asm volatile("ld.global.cg.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "l"(p));
  return v;
}
__device__ __forceinline__ float4 ld_cg4(const float4* p) {
  float4 v;
  asm volatile("ld.global.cg.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}

struct MergeParams {
  Ws ws;
  void* out;
  float* lse;                // optional [B][T][Hq] log-sum-exp of each output row
  int S, Hkv, G, Hq, slots;  // slots = 2 * V partial slots in the workspace
  int T, GT;                 // query tokens per sequence; rows per segment = G * T
};

// LIST: the plan was made inside the decode kernel, which also listed the
// split segments with their descriptors (Ws::mlist, its count in the header
// under the step's parity); only those are visited.  Otherwise every segment
// is.  A job's loads form a chain (list count, list entry, partials), so it
// is kept short: the counts and the parity come in one 16-byte load.
template <int D, bool OUT_F32, bool LIST>
__global__ void __launch_bounds__(kMergeWarps * 32) merge_kernel(const MergeParams p) {
  constexpr int kVec = D / 32;                 // output elements per lane
  constexpr int kBatch = D == 128 ? 24 : 32;   // pieces loaded together (<= 32)
  pdl_wait();                                  // the partials of the decode kernel
  const int G = p.GT, lane = threadIdx.x & 31;  // rows per segment
  int nseg = p.S;
  if constexpr (LIST) {
    // header words kHdrListCount (two counts, by parity) and kHdrParity, at a
    // 16-byte boundary; the decode kernel before this merge flipped the
    // parity on its way out
    static_assert(kHdrListCount % 4 == 0 && kHdrParity == kHdrListCount + 2, "header words");
    const int4 lc = __ldcg(reinterpret_cast<const int4*>(p.ws.header + kHdrListCount));
    nseg = (lc.z & 1) ? lc.x : lc.y;
    if (nseg < 0 || nseg > p.S) {
      if (threadIdx.x == 0) atomicOr(&p.ws.header[kHdrStatus], HPA_DEVICE_BAD_PLAN);
      nseg = 0;
    }
  }
  const int jobs = nseg * G;
  for (int job = blockIdx.x * kMergeWarps + (threadIdx.x >> 5); job < jobs;
       job += gridDim.x * kMergeWarps) {
    const int k = job / G, h = job - k * G;
    int s = k;
    int2 sd;
    if constexpr (LIST) {
      const int4 ent = __ldcg(&p.ws.mlist[k]);
      s = ent.x;
      sd = make_int2(ent.y, ent.z);
    }
    if (s < 0 || s >= p.S) {
      if (lane == 0) atomicOr(&p.ws.header[kHdrStatus], HPA_DEVICE_BAD_PLAN);
      continue;
    }
    if constexpr (!LIST) sd = __ldcg(&p.ws.seg_desc[s]);
    const int ns = sd.y;
    if (ns <= 1) continue;
    const int r0 = sd.x >> 1;
    if (sd.x < 0 || 2LL * (r0 + ns - 1) >= p.slots) {
      if (lane == 0) atomicOr(&p.ws.header[kHdrStatus], HPA_DEVICE_BAD_PLAN);
      continue;
    }
    // piece i sits in slot sd.x (i = 0), else 2 (r0 + i)
    auto row = [&](int i) -> long long { return (i == 0 ? (long long)sd.x : 2LL * (r0 + i)) * G + h; };
    float M = -INFINITY, lam = 0.f, o[kVec];
#pragma unroll
    for (int v = 0; v < kVec; ++v) o[v] = 0.f;
    for (int i0 = 0; i0 < ns; i0 += kBatch) {
      const int n = min(kBatch, ns - i0);
      const float2 ml = lane < n ? ld_cg2(p.ws.part_ml + row(i0 + lane)) : make_float2(-INFINITY, 0.f);
      float a[kBatch][kVec];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const float* src = p.ws.part_acc + row(i0 + j) * D + lane * kVec;
        if constexpr (kVec == 4) {
          const float4 x = j < n ? ld_cg4(reinterpret_cast<const float4*>(src)) : make_float4(0.f, 0.f, 0.f, 0.f);
          a[j][0] = x.x; a[j][1] = x.y; a[j][2] = x.z; a[j][3] = x.w;
        } else {
          const float2 x = j < n ? ld_cg2(reinterpret_cast<const float2*>(src)) : make_float2(0.f, 0.f);
          a[j][0] = x.x; a[j][1] = x.y;
        }
      }
      float Mn = ml.x;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) Mn = fmaxf(Mn, __shfl_xor_sync(0xffffffffu, Mn, off));
      Mn = fmaxf(M, Mn);
      const float w = (ml.x == -INFINITY) ? 0.f : fast_exp2(ml.x - Mn);
      const float sc = (M == -INFINITY) ? 0.f : fast_exp2(M - Mn);
      float lw = ml.y * w;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) lw += __shfl_xor_sync(0xffffffffu, lw, off);
      lam = lam * sc + lw;
#pragma unroll
      for (int v = 0; v < kVec; ++v) o[v] *= sc;
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const float wj = __shfl_sync(0xffffffffu, w, j);
#pragma unroll
        for (int v = 0; v < kVec; ++v) o[v] += a[j][v] * wj;
      }
      M = Mn;
    }
    const float inv = lam > 0.f ? 1.f / lam : 0.f;  // a row that sees no token is 0
#pragma unroll
    for (int v = 0; v < kVec; ++v) o[v] *= inv;
    const int b = s / p.Hkv, g = s - b * p.Hkv;
    const int qi = h / p.G, hh = h - qi * p.G;  // row h = query token qi, head hh
    const long long orow = ((long long)b * p.T + qi) * p.Hq + (long long)g * p.G + hh;
    store_out_vec<OUT_F32, kVec>(p.out, orow * D + lane * kVec, o);
    if (p.lse && lane == 0) p.lse[orow] = lse_of(M, lam);
  }
  pdl_trigger();
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// A cache viewed as a 2-D tensor [num_pages * Hkv * 64 rows][D]; one box is 64
// rows x 128 bytes with 128-byte swizzle.
bool encode_cache_map(CUtensorMap* tm, const void* base, int num_pages, int Hkv, int D, bool fp8) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const int elt = fp8 ? 1 : 2;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)num_pages * Hkv * kPageSize};
  cuuint64_t strides[1] = {(cuuint64_t)D * elt};
  cuuint32_t box[2] = {(cuuint32_t)(128 / elt), (cuuint32_t)kPageSize};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(tm, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The same caches come back every decode step: keep the last few maps per
// host thread, keyed by everything the map encodes, instead of encoding two
// maps per call.
bool make_cache_map(CUtensorMap* tm, const void* base, int num_pages, int Hkv, int D, bool fp8) {
  struct Entry {
    const void* base;
    int num_pages, Hkv, D;
    bool fp8, used;
    CUtensorMap map;
  };
  constexpr int kEntries = 8;
  thread_local Entry cache[kEntries] = {};
  thread_local int next = 0;
  for (const Entry& e : cache)
    if (e.used && e.base == base && e.num_pages == num_pages && e.Hkv == Hkv && e.D == D &&
        e.fp8 == fp8) {
      *tm = e.map;
      return true;
    }
  if (!encode_cache_map(tm, base, num_pages, Hkv, D, fp8)) return false;
  Entry& e = cache[next];
  next = (next + 1) % kEntries;
  e = Entry{base, num_pages, Hkv, D, fp8, true, *tm};
  return true;
}

template <int D, int NT, bool FP8, bool OUT_F32, int CPS, bool PRO, bool FP>
hpa_status launch(const CUtensorMap& tk, const CUtensorMap& tv, const RunParams& p, int grid,
                  cudaStream_t stream) {
  using C = Cfg<D, NT, FP8, CPS, PRO, FP>;
  auto kern = decode_kernel<D, NT, FP8, OUT_F32, CPS, PRO, FP>;
  // The shared-memory opt-in is per device; remember which devices have it.
  static std::atomic<uint64_t> ready_mask{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    set_cuda_error(e, "hpa_decode_run cudaGetDevice");
    return HPA_ERR_CUDA;
  }
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
  if (!bit || !(ready_mask.load() & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) {
      set_cuda_error(e, "hpa_decode_run smem attribute");
      return HPA_ERR_CUDA;
    }
    ready_mask.fetch_or(bit);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tk, tv, p);
  if (e != cudaSuccess) {
    set_cuda_error(e, "hpa_decode_run launch");
    return HPA_ERR_CUDA;
  }
  return HPA_OK;
}

// One persistent CTA per SM when the grid fits the SMs; two co-resident
// (smaller) CTAs per SM when the grid is larger, so that twice as many
// consumer warps hide each other's latencies.
template <int D, bool FP8, bool OUT_F32, bool PRO, bool FP>
hpa_status launch_nt(int nt, int cps, const CUtensorMap& tk, const CUtensorMap& tv,
                     const RunParams& p, int grid, cudaStream_t s) {
  if constexpr (!PRO) {
    // 17..32 rows (multi-token only)
    if (nt == 4)
      return cps == 2 ? launch<D, 4, FP8, OUT_F32, 2, PRO, FP>(tk, tv, p, grid, s)
                      : launch<D, 4, FP8, OUT_F32, 1, PRO, FP>(tk, tv, p, grid, s);
  }
  if (cps == 1)
    return nt == 1 ? launch<D, 1, FP8, OUT_F32, 1, PRO, FP>(tk, tv, p, grid, s)
                   : launch<D, 2, FP8, OUT_F32, 1, PRO, FP>(tk, tv, p, grid, s);
  return nt == 1 ? launch<D, 1, FP8, OUT_F32, 2, PRO, FP>(tk, tv, p, grid, s)
                 : launch<D, 2, FP8, OUT_F32, 2, PRO, FP>(tk, tv, p, grid, s);
}

template <bool OUT_F32, bool PRO, bool FP>
hpa_status launch_d(bool fp8, int head_dim, int nt, int cps, const CUtensorMap& tk,
                    const CUtensorMap& tv, const RunParams& p, int grid, cudaStream_t s) {
  if constexpr (!PRO) {
    if (fp8) return launch_nt<128, true, OUT_F32, false, FP>(nt, cps, tk, tv, p, grid, s);
  }
  return head_dim == 128 ? launch_nt<128, false, OUT_F32, PRO, FP>(nt, cps, tk, tv, p, grid, s)
                         : launch_nt<64, false, OUT_F32, PRO, FP>(nt, cps, tk, tv, p, grid, s);
}

// Arguments of the fused prologue (hpa_decode_run_prologue).
struct ProArgs {
  const void *k_raw, *v_raw;
  const float *q_gamma, *k_gamma;
  float eps, rope_theta;
  void* q_out;
};

// Cached SM count of the current device (0 if unknown).
int sm_count() {
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

// Validation, parameters and launches shared by hpa_decode_run and
// hpa_decode_run_prologue (pro != nullptr: q is the raw query).
hpa_status run_impl(const void* q, const void* k_cache, const void* v_cache, const float* k_scale,
                    const float* v_scale, hpa_kv_dtype kv_dtype, const int32_t* page_table,
                    int pt_stride, int num_pages, void* out, hpa_out_dtype out_dtype, int batch,
                    int num_q_heads, int num_kv_heads, int head_dim, float softmax_scale,
                    hpa_plan_kind kind, int grid, void* workspace, size_t ws_bytes, void* stream,
                    const ProArgs* pro, int q_tokens, const int32_t* plan_lens,
                    float* lse = nullptr) {
  if (!q || !k_cache || !v_cache || !page_table || !out || !workspace) return HPA_ERR_INVALID_ARG;
  if (batch <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || pt_stride <= 0 || num_pages <= 0 ||
      grid <= 0)
    return HPA_ERR_INVALID_ARG;
  if (num_q_heads % num_kv_heads) return HPA_ERR_INVALID_ARG;
  if (kv_dtype != HPA_KV_BF16 && kv_dtype != HPA_KV_FP8_E4M3) return HPA_ERR_INVALID_ARG;
  if (out_dtype != HPA_OUT_BF16 && out_dtype != HPA_OUT_F32) return HPA_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return HPA_ERR_INVALID_ARG;
  const bool fp8 = kv_dtype == HPA_KV_FP8_E4M3;
  if (fp8 && (!k_scale || !v_scale)) return HPA_ERR_INVALID_ARG;
  const int G = num_q_heads / num_kv_heads;
  if (G > 32) return HPA_ERR_UNSUPPORTED;  // a kv head's rows fill at most four MMA n-tiles
  if (q_tokens < 1) return HPA_ERR_INVALID_ARG;
  // the G * T rows of a kv head ride on the MMA N dimension: at most 32
  if (q_tokens > kMaxQTokens || G * q_tokens > 32) return HPA_ERR_UNSUPPORTED;
  // the fused prologue: one query token, at most two n-tiles
  if (pro && (q_tokens != 1 || G > 16)) return HPA_ERR_UNSUPPORTED;
  if (plan_lens) {
    // in-kernel plan: the dynamic plan for `grid` persistent CTAs, with the
    // plan kernel's limits and the tile offsets in shared memory
    if (kind != HPA_PLAN_DYNAMIC) return HPA_ERR_INVALID_ARG;
    if (batch > kMaxFusedBatch || grid > 65536) return HPA_ERR_UNSUPPORTED;
    if ((long long)pt_stride * kPageSize > 0x7fffffffLL) return HPA_ERR_UNSUPPORTED;
    if ((long long)batch * pt_stride * num_kv_heads > 0x7fffffffLL) return HPA_ERR_UNSUPPORTED;
  }
  const int GT = G * q_tokens;
  if (head_dim != 64 && head_dim != 128) return HPA_ERR_UNSUPPORTED;
  if (fp8 && head_dim != 128) return HPA_ERR_UNSUPPORTED;
  if ((long long)num_pages * num_kv_heads * kPageSize > 0x7fffffffLL) return HPA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache)) & 15)
    return HPA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q) & 15) || (reinterpret_cast<uintptr_t>(out) & 3))
    return HPA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(lse) & 3) return HPA_ERR_INVALID_ARG;
  if (pro) {
    if (!pro->k_raw || !pro->v_raw || !pro->q_gamma || !pro->k_gamma) return HPA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(pro->k_raw) | reinterpret_cast<uintptr_t>(pro->v_raw)) & 15)
      return HPA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(pro->q_out) & 1) return HPA_ERR_INVALID_ARG;
    if (!(pro->eps >= 0.f) || !std::isfinite(pro->eps) || !(pro->rope_theta > 0.f) ||
        !std::isfinite(pro->rope_theta))
      return HPA_ERR_INVALID_ARG;
    if (fp8) return HPA_ERR_UNSUPPORTED;  // the new row would need a new page scale
  }
  WsLayout L;
  // the plan and workspace of a multi-token step count G * T rows per kv head
  if (!ws_layout(kind, batch, num_kv_heads, num_q_heads * q_tokens, head_dim, grid, &L))
    return HPA_ERR_INVALID_ARG;
  if (ws_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255)) return HPA_ERR_WORKSPACE;

  CUtensorMap tk, tv;
  if (!make_cache_map(&tk, k_cache, num_pages, num_kv_heads, head_dim, fp8) ||
      !make_cache_map(&tv, v_cache, num_pages, num_kv_heads, head_dim, fp8)) {
    set_cuda_error(cudaErrorInvalidValue, "cuTensorMapEncodeTiled");
    return HPA_ERR_CUDA;
  }
  RunParams p;
  p.q = static_cast<const uint16_t*>(q);
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.page_table = page_table;
  p.pt_stride = pt_stride;
  p.num_pages = num_pages;
  p.out = out;
  p.lse = lse;
  p.B = batch;
  p.Hq = num_q_heads;
  p.Hkv = num_kv_heads;
  p.G = G;
  p.T = q_tokens;
  p.GT = GT;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.ws = ws_view(workspace, L);
  p.grid = grid;
  p.kind = kind;
  p.slots = (int)(2 * plan_ranges_ll(kind, grid));
  p.k_raw = pro ? static_cast<const __nv_bfloat16*>(pro->k_raw) : nullptr;
  p.v_raw = pro ? static_cast<const __nv_bfloat16*>(pro->v_raw) : nullptr;
  p.q_gamma = pro ? pro->q_gamma : nullptr;
  p.k_gamma = pro ? pro->k_gamma : nullptr;
  p.eps = pro ? pro->eps : 0.f;
  p.log2_theta = pro ? std::log2((double)pro->rope_theta) : 0.0;
  p.k_cache_w = pro ? static_cast<__nv_bfloat16*>(const_cast<void*>(k_cache)) : nullptr;
  p.v_cache_w = pro ? static_cast<__nv_bfloat16*>(const_cast<void*>(v_cache)) : nullptr;
  p.q_out = pro ? static_cast<__nv_bfloat16*>(pro->q_out) : nullptr;
  p.seq_lens = plan_lens;
  p.capacity = pt_stride * kPageSize;
  p.tail_den = HPA_TAIL_DEN_DEFAULT;
  p.tail_chunks = HPA_TAIL_CHUNKS_DEFAULT;
  p.tail_min = HPA_TAIL_MIN_DEFAULT;
  p.unit_cost = HPA_COST_UNIT_DEFAULT;
  p.end_cost = fp8 ? HPA_COST_END_DEFAULT_FP8 : HPA_COST_END_DEFAULT;
  const int nt = GT > 16 ? 4 : GT > 8 ? 2 : 1;
  const int sms = sm_count();
  const int cps = (sms > 0 && grid > sms) ? 2 : 1;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool f32 = out_dtype == HPA_OUT_F32;
  hpa_status st;
  if (pro && plan_lens)
    st = f32 ? launch_d<true, true, true>(fp8, head_dim, nt, cps, tk, tv, p, grid, s)
             : launch_d<false, true, true>(fp8, head_dim, nt, cps, tk, tv, p, grid, s);
  else if (pro)
    st = f32 ? launch_d<true, true, false>(fp8, head_dim, nt, cps, tk, tv, p, grid, s)
             : launch_d<false, true, false>(fp8, head_dim, nt, cps, tk, tv, p, grid, s);
  else if (plan_lens)
    st = f32 ? launch_d<true, false, true>(fp8, head_dim, nt, cps, tk, tv, p, grid, s)
             : launch_d<false, false, true>(fp8, head_dim, nt, cps, tk, tv, p, grid, s);
  else
    st = f32 ? launch_d<true, false, false>(fp8, head_dim, nt, cps, tk, tv, p, grid, s)
             : launch_d<false, false, false>(fp8, head_dim, nt, cps, tk, tv, p, grid, s);
  if (st != HPA_OK) return st;

  // split merge, chained behind the decode kernel
  MergeParams mp;
  mp.ws = p.ws;
  mp.out = out;
  mp.lse = lse;
  mp.S = batch * num_kv_heads;
  mp.Hkv = num_kv_heads;
  mp.G = G;
  mp.T = q_tokens;
  mp.GT = GT;
  mp.Hq = num_q_heads;
  mp.slots = (int)(2 * plan_ranges_ll(kind, grid));
  cudaLaunchConfig_t cfg = {};
  const long long merge_ctas = ((long long)mp.S * GT + kMergeWarps - 1) / kMergeWarps;
  // with the split segments listed (in-kernel plan), fewer CTAs: most
  // segments need no merge
  const long long cap = (long long)std::max(1, sms) * (plan_lens ? 8 : 16);
  cfg.gridDim = dim3((unsigned)std::min<long long>(merge_ctas, cap));
  cfg.blockDim = dim3(kMergeWarps * 32);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (plan_lens) {
    if (head_dim == 128)
      e = f32 ? cudaLaunchKernelEx(&cfg, merge_kernel<128, true, true>, mp)
              : cudaLaunchKernelEx(&cfg, merge_kernel<128, false, true>, mp);
    else
      e = f32 ? cudaLaunchKernelEx(&cfg, merge_kernel<64, true, true>, mp)
              : cudaLaunchKernelEx(&cfg, merge_kernel<64, false, true>, mp);
  } else {
    if (head_dim == 128)
      e = f32 ? cudaLaunchKernelEx(&cfg, merge_kernel<128, true, false>, mp)
              : cudaLaunchKernelEx(&cfg, merge_kernel<128, false, false>, mp);
    else
      e = f32 ? cudaLaunchKernelEx(&cfg, merge_kernel<64, true, false>, mp)
              : cudaLaunchKernelEx(&cfg, merge_kernel<64, false, false>, mp);
  }
  if (e != cudaSuccess) {
    set_cuda_error(e, "hpa_decode_run merge launch");
    return HPA_ERR_CUDA;
  }
  return HPA_OK;
}

}  // namespace
}  // namespace hpa

extern "C" hpa_status hpa_decode_run(const void* q, const void* k_cache, const void* v_cache,
                                     const float* k_scale, const float* v_scale,
                                     hpa_kv_dtype kv_dtype, const int32_t* page_table,
                                     int pt_stride, int num_pages, void* out,
                                     hpa_out_dtype out_dtype, int batch, int num_q_heads,
                                     int num_kv_heads, int head_dim, float softmax_scale,
                                     hpa_plan_kind kind, int grid, void* workspace,
                                     size_t ws_bytes, void* stream) {
  return hpa::run_impl(q, k_cache, v_cache, k_scale, v_scale, kv_dtype, page_table, pt_stride,
                       num_pages, out, out_dtype, batch, num_q_heads, num_kv_heads, head_dim,
                       softmax_scale, kind, grid, workspace, ws_bytes, stream, nullptr, 1, nullptr);
}

extern "C" hpa_status hpa_decode_run_multi(const void* q, const void* k_cache, const void* v_cache,
                                           const float* k_scale, const float* v_scale,
                                           hpa_kv_dtype kv_dtype, const int32_t* page_table,
                                           int pt_stride, int num_pages, void* out,
                                           hpa_out_dtype out_dtype, int batch, int q_tokens,
                                           int num_q_heads, int num_kv_heads, int head_dim,
                                           float softmax_scale, hpa_plan_kind kind, int grid,
                                           void* workspace, size_t ws_bytes, void* stream) {
  return hpa::run_impl(q, k_cache, v_cache, k_scale, v_scale, kv_dtype, page_table, pt_stride,
                       num_pages, out, out_dtype, batch, num_q_heads, num_kv_heads, head_dim,
                       softmax_scale, kind, grid, workspace, ws_bytes, stream, nullptr, q_tokens,
                       nullptr);
}

extern "C" hpa_status hpa_decode_step(const int32_t* seq_lens, const void* q, const void* k_cache,
                                      const void* v_cache, const float* k_scale,
                                      const float* v_scale, hpa_kv_dtype kv_dtype,
                                      const int32_t* page_table, int pt_stride, int num_pages,
                                      void* out, hpa_out_dtype out_dtype, int batch, int q_tokens,
                                      int num_q_heads, int num_kv_heads, int head_dim,
                                      float softmax_scale, int num_ctas, void* workspace,
                                      size_t ws_bytes, void* stream) {
  if (!seq_lens) return HPA_ERR_INVALID_ARG;
  return hpa::run_impl(q, k_cache, v_cache, k_scale, v_scale, kv_dtype, page_table, pt_stride,
                       num_pages, out, out_dtype, batch, num_q_heads, num_kv_heads, head_dim,
                       softmax_scale, HPA_PLAN_DYNAMIC, num_ctas, workspace, ws_bytes, stream,
                       nullptr, q_tokens, seq_lens);
}

extern "C" hpa_status hpa_decode_run_prologue(
    const void* q_raw, const void* k_raw, const void* v_raw, const float* q_gamma,
    const float* k_gamma, float eps, float rope_theta, void* k_cache, void* v_cache, void* q_out,
    const int32_t* page_table, int pt_stride, int num_pages, void* out, hpa_out_dtype out_dtype,
    int batch, int num_q_heads, int num_kv_heads, int head_dim, float softmax_scale,
    hpa_plan_kind kind, int grid, void* workspace, size_t ws_bytes, void* stream) {
  const hpa::ProArgs pro{k_raw, v_raw, q_gamma, k_gamma, eps, rope_theta, q_out};
  return hpa::run_impl(q_raw, k_cache, v_cache, nullptr, nullptr, HPA_KV_BF16, page_table,
                       pt_stride, num_pages, out, out_dtype, batch, num_q_heads, num_kv_heads,
                       head_dim, softmax_scale, kind, grid, workspace, ws_bytes, stream, &pro, 1,
                       nullptr);
}

extern "C" hpa_status hpa_decode_step_prologue(
    const int32_t* seq_lens, const void* q_raw, const void* k_raw, const void* v_raw,
    const float* q_gamma, const float* k_gamma, float eps, float rope_theta, void* k_cache,
    void* v_cache, void* q_out, const int32_t* page_table, int pt_stride, int num_pages,
    void* out, hpa_out_dtype out_dtype, int batch, int num_q_heads, int num_kv_heads,
    int head_dim, float softmax_scale, int num_ctas, void* workspace, size_t ws_bytes,
    void* stream) {
  if (!seq_lens) return HPA_ERR_INVALID_ARG;
  const hpa::ProArgs pro{k_raw, v_raw, q_gamma, k_gamma, eps, rope_theta, q_out};
  return hpa::run_impl(q_raw, k_cache, v_cache, nullptr, nullptr, HPA_KV_BF16, page_table,
                       pt_stride, num_pages, out, out_dtype, batch, num_q_heads, num_kv_heads,
                       head_dim, softmax_scale, HPA_PLAN_DYNAMIC, num_ctas, workspace, ws_bytes,
                       stream, &pro, 1, seq_lens);
}

extern "C" hpa_status hpa_decode_step_lse(const int32_t* seq_lens, const void* q,
                                          const void* k_cache, const void* v_cache,
                                          const float* k_scale, const float* v_scale,
                                          hpa_kv_dtype kv_dtype, const int32_t* page_table,
                                          int pt_stride, int num_pages, void* out,
                                          hpa_out_dtype out_dtype, float* lse, int batch,
                                          int q_tokens, int num_q_heads, int num_kv_heads,
                                          int head_dim, float softmax_scale, int num_ctas,
                                          void* workspace, size_t ws_bytes, void* stream) {
  if (!seq_lens || !lse) return HPA_ERR_INVALID_ARG;
  return hpa::run_impl(q, k_cache, v_cache, k_scale, v_scale, kv_dtype, page_table, pt_stride,
                       num_pages, out, out_dtype, batch, num_q_heads, num_kv_heads, head_dim,
                       softmax_scale, HPA_PLAN_DYNAMIC, num_ctas, workspace, ws_bytes, stream,
                       nullptr, q_tokens, seq_lens, lse);
}
