// hpa_common.cuh -- shared pieces of the sm_100a kernels: the workspace layout,
// inline-PTX wrappers (mbarrier, TMA, ldmatrix/movmatrix, mma.sync, PDL) and
// small host helpers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hpa.h"

namespace hpa {

constexpr int kPageSize = 64;            // tokens per page == tokens per tile
constexpr int kMaxPlanBatch = 32768;     // sequences per plan (tile offsets live in shared memory)
constexpr int kMaxFusedBatch = 512;      // sequences an in-kernel plan keeps in shared memory
constexpr int32_t kPlanMagic = 0x31415048;  // "HPA1"

// ---------------------------------------------------------------------------
// Workspace layout.  Every region starts on a 256-byte boundary.
//   header      int32[32]: magic, status, U, grid, kind, B, Hkv, G, D, T, V, next, done,
//                          tail_den, tail_chunks, tail_min, split segments listed
//                          (two counts, by step parity), the step parity (the
//                          run-time counters sit in the header, at the same
//                          offset for every layout)
//   lens        int32[B]     clamped lengths
//   tile_start  int32[B+1]   exclusive prefix sum of tiles per sequence
//   cta_desc    int4[2*V]    per range v: (u_begin, u_end, b0, g0), (t0, n0,
//                            0, 0): the unit range and the (sequence, kv
//                            head, tile, tiles of that sequence) of its first
//                            unit.  V = grid for the static plans; for the
//                            dynamic plan V <= 5 * grid (grid primary ranges,
//                            then the tail chunks).
//   seg_desc    int2[B*Hkv]  per segment: (first partial slot, ranges holding
//                            its units); a segment held by one range has no
//                            partials.
//   mlist       int4[B*Hkv]  in-kernel plan: the split segments, each as (id,
//                            first partial slot, ranges holding it, 0), in
//                            no particular order (their count is in the
//                            header); the merge kernel visits only them.  A
//                            step appends to the count of its parity; its last
//                            CTA zeroes the other count (the previous step's,
//                            whose merge has finished) and flips the parity
//   part_ml     float2[2V][G]     (m, l) of each partial, log2 units
//   part_acc    float[2V][G][D]   un-normalised partial outputs
//   trace       uint64[grid][4]   per run-kernel CTA: %globaltimer (ns) at its
//                                 start, when its producer ran out of work and
//                                 when its epilogue finished; units it streamed
// Partial slots follow from the ranges: range v stores the piece of its first
// segment in slot 2v and the piece of its last segment in slot 2v + 1 (a
// segment in the middle of a range is whole there).  The ranges holding a
// segment are consecutive, r0 .. r0 + n - 1; the segment's piece in r0 is
// in slot 2 r0 (if the segment starts where r0 does) or 2 r0 + 1, and its
// piece in each later range r is in slot 2r.
// ---------------------------------------------------------------------------
enum HeaderField {
  kHdrMagic = 0, kHdrStatus = 1, kHdrUnits = 2, kHdrGrid = 3, kHdrKind = 4,
  kHdrBatch = 5, kHdrKvHeads = 6, kHdrGroup = 7, kHdrHeadDim = 8, kHdrTiles = 9,
  kHdrRanges = 10,  // virtual ranges V (grid for static plans)
  kHdrNext = 11,    // dynamic plan: next tail chunk to hand out (run-time counter)
  kHdrDone = 12,    // in-kernel plan: CTAs of the current step that finished
  kHdrTailDen = 13,     // dynamic plans: the tail parameters the plan was made with
  kHdrTailChunks = 14,
  kHdrTailMin = 15,
  kHdrListCount = 16,   // in-kernel plan: split segments on the merge list (2 words: by parity)
  kHdrParity = 18,      // in-kernel plan: parity of the current step
  kHdrUnitCost = 19,    // dynamic plans: the cost weights of the primary cuts
  kHdrEndCost = 20,
  kHdrWords = 32
};

// The dynamic plan gives each of its P persistent CTAs one primary range and
// hands out up to tail_chunks * P tail chunks at run time (tail_chunks <=
// HPA_TAIL_CHUNKS_MAX, which sizes the workspace).
constexpr int kMaxTailChunksPerCta = HPA_TAIL_CHUNKS_MAX;
constexpr int kLaDefaultMinPiece = 4;  // LENGTH_AWARE: smallest piece of a cut segment, tiles

#if defined(__CUDACC__)
#define HPA_HD __host__ __device__
#else
#define HPA_HD
#endif

// DYNAMIC and LENGTH_AWARE: P primary ranges + up to 4P run-time tail chunks
// (HPA_TAIL_CHUNKS_MAX per CTA)
HPA_HD inline bool plan_is_dynamic(int kind) {
  return kind == HPA_PLAN_DYNAMIC || kind == HPA_PLAN_LENGTH_AWARE;
}

// Virtual ranges a plan of this kind and grid can describe.
HPA_HD inline long long plan_ranges_ll(int kind, int grid) {
  return plan_is_dynamic(kind) ? (long long)grid * (1 + kMaxTailChunksPerCta) : grid;
}

struct WsLayout {
  size_t header, lens, tile_start, cta_desc, seg_desc, mlist, part_ml, part_acc, trace, total;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline bool ws_layout(int kind, int B, int Hkv, int Hq, int D, int grid, WsLayout* L) {
  if (B <= 0 || Hkv <= 0 || Hq <= 0 || D <= 0 || grid <= 0 || Hq % Hkv) return false;
  if (kind != HPA_PLAN_DYNAMIC && kind != HPA_PLAN_STATIC_NSPLIT && kind != HPA_PLAN_STATIC_CHUNK &&
      kind != HPA_PLAN_LENGTH_AWARE)
    return false;
  const size_t V = size_t(plan_ranges_ll(kind, grid));
  const size_t G = size_t(Hq / Hkv), S = size_t(B) * Hkv, slots = 2 * V;
  size_t off = 0;
  L->header = off;      off = align256(off + kHdrWords * 4);
  L->lens = off;        off = align256(off + size_t(B) * 4);
  L->tile_start = off;  off = align256(off + (size_t(B) + 1) * 4);
  L->cta_desc = off;    off = align256(off + V * 32);
  L->seg_desc = off;    off = align256(off + S * 8);
  L->mlist = off;       off = align256(off + S * 16);
  L->part_ml = off;     off = align256(off + slots * G * 8);
  L->part_acc = off;    off = align256(off + slots * G * size_t(D) * 4);
  L->trace = off;       off = align256(off + size_t(grid) * 32);
  L->total = off;
  return true;
}

// Device view of a workspace.
struct Ws {
  int32_t* header;
  int32_t* lens;
  int32_t* tile_start;
  int4* cta_desc;
  int2* seg_desc;
  int4* mlist;
  float2* part_ml;
  float* part_acc;
  unsigned long long* trace;
};

inline Ws ws_view(void* base, const WsLayout& L) {
  char* p = static_cast<char*>(base);
  return Ws{reinterpret_cast<int32_t*>(p + L.header), reinterpret_cast<int32_t*>(p + L.lens),
            reinterpret_cast<int32_t*>(p + L.tile_start), reinterpret_cast<int4*>(p + L.cta_desc),
            reinterpret_cast<int2*>(p + L.seg_desc), reinterpret_cast<int4*>(p + L.mlist),
            reinterpret_cast<float2*>(p + L.part_ml),
            reinterpret_cast<float*>(p + L.part_acc),
            reinterpret_cast<unsigned long long*>(p + L.trace)};
}

// Host-side grid of a plan (must equal the oracle's definition; see hpa.h).
inline long long plan_grid_ll(int kind, int B, int Hkv, int num_ctas, int param,
                              int max_seq_len, long long* chunk_out) {
  if (B <= 0 || Hkv <= 0 || num_ctas <= 0 || param < 0 || max_seq_len < 0) return -1;
  if (chunk_out) *chunk_out = 0;
  if (plan_is_dynamic(kind)) return num_ctas;
  const long long S = (long long)B * Hkv;
  if (kind == HPA_PLAN_STATIC_NSPLIT) {
    long long s = param > 0 ? param : (num_ctas + S - 1) / S;
    if (s < 1) s = 1;
    return S * s;
  }
  if (kind == HPA_PLAN_STATIC_CHUNK) {
    const long long tmax = ((long long)max_seq_len + kPageSize - 1) / kPageSize;
    const long long per_seg = (num_ctas + Hkv - 1) / Hkv;
    long long c = param > 0 ? param : (tmax + per_seg - 1) / per_seg;
    if (c < 1) c = 1;
    long long nc = (tmax + c - 1) / c;
    if (nc < 1) nc = 1;
    if (chunk_out) *chunk_out = c;
    return S * nc;
  }
  return -1;
}

// Records a CUDA error for hpa_last_cuda_error().
void set_cuda_error(cudaError_t e, const char* where);

// ---------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------
#if defined(__CUDACC__)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Programmatic dependent launch: wait for the preceding grid's memory, and let
// the next grid start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// 1-D bulk copy global -> shared (16-byte aligned, size a multiple of 16),
// completing on an mbarrier (no multicast).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* tm) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tm)) : "memory");
}

// 2-D TMA tile load global -> shared, completing on an mbarrier (no multicast).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* tm, int x, int y,
                                            uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// D = A(16x16, row) * B(16x8, col) + D, bf16 or f16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two fp32 -> packed bf16x2 / f16x2 (round to nearest even); `lo` in the low half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// Two e4m3 codes (low byte = first) -> f16x2 (exact: every e4m3 value is an f16).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t codes) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(codes));
  return r;
}

// Order this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (TMA / bulk copy) accesses to the same memory.
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

#endif  // __CUDACC__

}  // namespace hpa
