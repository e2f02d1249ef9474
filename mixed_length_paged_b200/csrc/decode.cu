// decode.cu -- persistent paged GQA decode attention (hpa_decode_run).
//
// The method (xiaodao.ai "HPC-Ops TPOT -48.8%", Attention section): persistent
// CTAs consume the planner's 64-token tile tasks; a (sequence, kv head) whose
// tiles span several CTAs is finished from per-split partials by a
// log-sum-exp merge.  The pages describe a Hopper design (TMA + WGMMA); this
// is written for sm_100a as follows.
//
// CTA = 4 consumer warps + 1 producer warp, one CTA per SM.
//   producer: walks the CTA's unit range, reads page ids (32 at a time, one
//     per lane), and for each unit issues 2-D TMA tile loads of the K and V
//     tiles of (page, kv head) -- each a contiguous 64 x D block -- into a
//     ring of shared-memory stages, with 128-byte swizzle so the tensor-core
//     fragment loads below are bank-conflict free.  Loads carry an L2
//     evict-first hint: the cache is streamed once per step.
//   consumers: warp w owns tokens [16w, 16w+16) of every tile and keeps its own
//     online-softmax state (m, l, acc) for the tile's G query heads:
//       S^T[16 tok x 8 heads] = K_w[16 x D] . Q^T        (mma m16n8k16, fp32 acc)
//       online softmax in base 2 (logits pre-scaled by scale * log2 e)
//       O^T[D x 8 heads]    += V_w^T[D x 16] . P^T      (P^T built in registers
//                                                       with movmatrix)
//     The GQA group sits on the MMA N dimension (8 heads per n-tile), so no
//     padding is needed for G = 8.  At the end of a (sequence, kv head)
//     segment the four warps' states are combined through shared memory; a
//     segment held whole by the CTA writes its output directly, otherwise the
//     CTA stores an (acc, m, l) partial and the last CTA to arrive merges all
//     partials of that segment in split order.
//
// FP8 (e4m3) caches: K/V codes are converted in registers with
// cvt.rn.f16x2.e4m3x2 (exact) and the products run as f16 MMAs; the
// per-(page, kv head) K scale folds into that tile's logits and the V scale
// into its probabilities.  To keep the e4m3 -> f16 conversion on whole
// registers, the D index inside each 16-wide MMA step is permuted (the same
// permutation on both operands, so the dot products are unchanged) and the
// output rows are un-permuted when stored.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>

#include <cuda_bf16.h>

#include "hpa_common.cuh"

namespace hpa {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kSmemLimit = 227 * 1024;
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s bound on any barrier wait

template <int D, int NT, bool FP8>
struct Cfg {
  static constexpr int kElt = FP8 ? 1 : 2;
  static constexpr int kRowBytes = D * kElt;           // one token row of one head
  static constexpr int kBoxes = kRowBytes / 128;       // 128-byte-wide TMA boxes per tile
  static constexpr int kBoxBytes = kPageSize * 128;    // 8 KiB
  static constexpr int kTileBytes = kPageSize * kRowBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;   // K tile + V tile
  static constexpr int kHeads = 8 * NT;                // MMA N (padded group)
  static constexpr int kAccStride = D + 4;             // floats; pads merge stores off one bank
  static constexpr int kMergeBytes = kConsumerWarps * kHeads * kAccStride * 4;
  static constexpr int kMlBytes = kConsumerWarps * kHeads * 8;
  static constexpr int kMisc = 1024;                   // barriers, stage info, flags
  static constexpr int kStagesFit = (kSmemLimit - 1024 - kMergeBytes - kMlBytes - kMisc) / kStageBytes;
  static constexpr int kStages = kStagesFit < 8 ? kStagesFit : 8;
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kMergeBytes + kMlBytes + kMisc;
  static constexpr int kKSteps = D / 16;               // QK MMA k-steps
  static constexpr int kMTiles = D / 16;               // PV MMA m-tiles
  static_assert(kRowBytes % 128 == 0, "tile rows must be whole 128-byte boxes");
  static_assert(kStages >= 2, "not enough shared memory for a pipeline");
};

struct RunParams {
  const uint16_t* q;        // bf16 bits [B][Hq][D]
  const float* k_scale;     // [pages][Hkv] (FP8)
  const float* v_scale;
  const int32_t* page_table;
  int pt_stride, num_pages;
  void* out;
  int B, Hq, Hkv, G;
  float scale_log2;         // softmax_scale * log2(e)
  Ws ws;
  int grid;
};

struct StageInfo {
  float k_scale, v_scale;
};

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

// Largest b in [0, B) with tile_start[b] * Hkv <= u.
__device__ __forceinline__ int seq_of_unit(const int32_t* ts, int B, int Hkv, int u) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((long long)ts[mid] * Hkv <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Walk over (b, g, t) units in global order.
struct Walk {
  int b, g, t, n;
  __device__ void init(const int32_t* ts, int B, int Hkv, int u) {
    b = seq_of_unit(ts, B, Hkv, u);
    n = ts[b + 1] - ts[b];
    const int rem = u - ts[b] * Hkv;
    g = rem / n;
    t = rem % n;
  }
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

// Shared-memory byte offset of 16-byte chunk `chunk` of token row `tok` in a
// tile stored as 128-byte-swizzled boxes of 64 rows x 128 bytes.
__device__ __forceinline__ uint32_t tile_addr(uint32_t tile, int tok, int chunk) {
  return tile + (chunk >> 3) * (kPageSize * 128) + tok * 128 + (((chunk & 7) ^ (tok & 7)) << 4);
}

template <int D, int NT, bool FP8, bool OUT_F32>
__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const RunParams p) {
  using C = Cfg<D, NT, FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  float* red_acc = reinterpret_cast<float*>(smem + C::kStages * C::kStageBytes);
  float2* red_ml = reinterpret_cast<float2*>(smem + C::kStages * C::kStageBytes + C::kMergeBytes);
  uint8_t* misc = smem + C::kStages * C::kStageBytes + C::kMergeBytes + C::kMlBytes;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(misc);
  uint64_t* empty_bar = full_bar + C::kStages;
  StageInfo* info = reinterpret_cast<StageInfo*>(empty_bar + C::kStages);
  volatile int* s_abort = reinterpret_cast<volatile int*>(info + C::kStages);
  volatile int* s_last = s_abort + 1;
  volatile int* s_plan_ok = s_abort + 2;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), kConsumerWarps);
    }
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == kConsumerWarps && lane == 0) {
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  // Everything below reads what the plan (and possibly the prologue) wrote.
  pdl_wait();
  if (threadIdx.x == 0) {
    const int32_t* h = p.ws.header;
    const bool ok = h[kHdrMagic] == kPlanMagic && h[kHdrGrid] == p.grid &&
                    h[kHdrGrid] == (int)gridDim.x && h[kHdrBatch] == p.B &&
                    h[kHdrKvHeads] == p.Hkv && h[kHdrGroup] == p.G && h[kHdrHeadDim] == D;
    *s_plan_ok = ok;
    if (!ok) atomicOr(&p.ws.header[kHdrStatus], HPA_DEVICE_BAD_PLAN);
  }
  __syncthreads();
  if (!*s_plan_ok) return;
  pdl_trigger();

  int32_t* status = &p.ws.header[kHdrStatus];
  const int32_t* ts = p.ws.tile_start;
  const int U = p.ws.header[kHdrUnits];
  const int4 desc = p.ws.cta_desc[blockIdx.x];
  const int ub = desc.x, ue = min(desc.y, U);

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    uint64_t policy = l2_policy_evict_first();
    Walk wk;
    int it = 0;
    if (ub < ue) wk.init(ts, p.B, p.Hkv, ub);
    for (int u0 = ub; u0 < ue; u0 += 32) {
      // lane i resolves unit u0 + i: (page, kv head) -> tile row, scales
      int row = 0, bad = 0;
      float ks = 1.f, vs = 1.f;
      {
        Walk w2 = wk;
        for (int k = 0; k < lane && u0 + k + 1 < ue; ++k) w2.next(ts, p.Hkv);
        if (u0 + lane < ue) {
          const int page = p.page_table[(long long)w2.b * p.pt_stride + w2.t];
          if (page < 0 || page >= p.num_pages) {
            bad = 1;
          } else {
            row = (page * p.Hkv + w2.g) * kPageSize;
            if constexpr (FP8) {
              ks = p.k_scale[page * p.Hkv + w2.g];
              vs = p.v_scale[page * p.Hkv + w2.g];
            }
          }
        }
      }
      const int cnt = min(32, ue - u0);
      for (int k = 0; k < cnt; ++k) {
        const int rk = __shfl_sync(0xffffffffu, row, k);
        const int bk = __shfl_sync(0xffffffffu, bad, k);
        const float kk = __shfl_sync(0xffffffffu, ks, k);
        const float vv = __shfl_sync(0xffffffffu, vs, k);
        if (lane == 0) {
          const int s = it % C::kStages;
          const uint32_t par = ((it / C::kStages) & 1) ^ 1;
          const uint32_t fb = smem_u32(&full_bar[s]);
          if (wait_bar(smem_u32(&empty_bar[s]), par, s_abort, status) && !bk) {
            info[s].k_scale = kk;
            info[s].v_scale = vv;
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
            if (bk) atomicOr(status, HPA_DEVICE_BAD_PAGE);
            mbar_arrive(fb);  // release consumers without data
          }
        }
        __syncwarp();
        ++it;
      }
      for (int k = 0; k < cnt; ++k)
        if (u0 + k + 1 < ue) wk.next(ts, p.Hkv);
    }
    // After an abort, make sure no copy is still landing in shared memory.
    if (lane == 0 && *s_abort) {
      const int first = max(0, it - C::kStages);
      for (int j = first; j < it; ++j) {
        const int s = j % C::kStages;
        const uint32_t fb = smem_u32(&full_bar[s]);
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(fb, (j / C::kStages) & 1) && globaltimer() - t0 < kWaitNs) {
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int r = lane >> 2, c = lane & 3;          // MMA fragment coordinates
  const int lm = lane >> 3, lr = lane & 7;        // ldmatrix address lane roles
  const int tok0 = warp * 16;                     // this warp's token slice
  // ldmatrix row (token) for the QK A operand and the PV A operand
  const int k_tok = tok0 + (lm & 1) * 8 + lr;
  const int k_chk = lm >> 1;
  const int v_tok = FP8 ? tok0 + (lm & 1) * 8 + lr : tok0 + (lm >> 1) * 8 + lr;
  const int v_chk = FP8 ? (lm >> 1) : (lm & 1);

  // zero output rows of empty sequences (a softmax over no tokens)
  for (int b = blockIdx.x; b < p.B; b += gridDim.x) {
    if (p.ws.lens[b] != 0) continue;
    for (int i = threadIdx.x; i < p.Hq * D; i += kConsumerWarps * 32) {
      const long long o = (long long)b * p.Hq * D + i;
      if constexpr (OUT_F32) reinterpret_cast<float*>(p.out)[o] = 0.f;
      else reinterpret_cast<__nv_bfloat16*>(p.out)[o] = __float2bfloat16_rn(0.f);
    }
  }

  uint32_t qf[NT][C::kKSteps][2];
  float acc[NT][C::kMTiles][4];
  float m_run[NT][2], l_run[NT][2];

  Walk wk;
  if (ub < ue) wk.init(ts, p.B, p.Hkv, ub);
  int seg_b = -1, seg_g = 0, L = 0;

  auto finish_segment = [&](int b, int g, int split_idx) {
    // full-warp l (m is already uniform across the lanes sharing a head)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float v = l_run[nt][e];
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        l_run[nt][e] = v;
      }
    float* my_acc = red_acc + warp * C::kHeads * C::kAccStride;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int h0 = nt * 8 + 2 * c;
#pragma unroll
      for (int i = 0; i < C::kMTiles; ++i) {
        const int d0 = FP8 ? 16 * i + 2 * r : 16 * i + r;
        const int d1 = FP8 ? d0 + 1 : d0 + 8;
        my_acc[h0 * C::kAccStride + d0] = acc[nt][i][0];
        my_acc[(h0 + 1) * C::kAccStride + d0] = acc[nt][i][1];
        my_acc[h0 * C::kAccStride + d1] = acc[nt][i][2];
        my_acc[(h0 + 1) * C::kAccStride + d1] = acc[nt][i][3];
      }
      if (r == 0) {
        red_ml[warp * C::kHeads + h0] = make_float2(m_run[nt][0], l_run[nt][0]);
        red_ml[warp * C::kHeads + h0 + 1] = make_float2(m_run[nt][1], l_run[nt][1]);
      }
    }
    named_bar_sync(1, kConsumerWarps * 32);

    const int s = b * p.Hkv + g;
    const int nsplit = p.ws.split_count[s];
    const int G = p.G;
    const int tid = threadIdx.x;
    const long long out_row0 = ((long long)b * p.Hq + (long long)g * G) * D;
    int slot = -1;
    if (nsplit > 1) {
      slot = p.ws.part_base[s] + split_idx;
      if (slot < 0 || slot >= 2 * p.grid || split_idx >= nsplit) {
        if (tid == 0) atomicOr(status, HPA_DEVICE_BAD_PLAN);
        slot = -1;
      }
    }
    for (int e = tid; e < G * D; e += kConsumerWarps * 32) {
      const int h = e / D, d = e - h * D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, red_ml[w * C::kHeads + h].x);
      float lam = 0.f, o = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float2 ml = red_ml[w * C::kHeads + h];
        const float sc = (ml.x == -INFINITY) ? 0.f : exp2f(ml.x - M);
        lam += ml.y * sc;
        o += red_acc[(w * C::kHeads + h) * C::kAccStride + d] * sc;
      }
      if (nsplit <= 1) {
        const float v = o / lam;
        if constexpr (OUT_F32) reinterpret_cast<float*>(p.out)[out_row0 + e] = v;
        else reinterpret_cast<__nv_bfloat16*>(p.out)[out_row0 + e] = __float2bfloat16_rn(v);
      } else if (slot >= 0) {
        p.ws.part_acc[((long long)slot * G + h) * D + d] = o;
        if (d == 0) p.ws.part_ml[(long long)slot * G + h] = make_float2(M, lam);
      }
    }
    if (nsplit > 1) {
      __threadfence();
      named_bar_sync(1, kConsumerWarps * 32);
      if (tid == 0) {
        const int prev = atomicAdd(&p.ws.arrive[s], 1);
        *s_last = (prev == nsplit - 1);
      }
      named_bar_sync(1, kConsumerWarps * 32);
      if (*s_last) {
        __threadfence();
        const int base = p.ws.part_base[s];
        if (base >= 0 && base + nsplit <= 2 * p.grid) {
          for (int e = tid; e < G * D; e += kConsumerWarps * 32) {
            const int h = e / D, d = e - h * D;
            float M = -INFINITY;
            for (int i = 0; i < nsplit; ++i)
              M = fmaxf(M, __ldcg(&p.ws.part_ml[(long long)(base + i) * G + h]).x);
            float lam = 0.f, o = 0.f;
            for (int i = 0; i < nsplit; ++i) {
              const float2 ml = __ldcg(&p.ws.part_ml[(long long)(base + i) * G + h]);
              const float sc = (ml.x == -INFINITY) ? 0.f : exp2f(ml.x - M);
              lam += ml.y * sc;
              o += __ldcg(&p.ws.part_acc[((long long)(base + i) * G + h) * D + d]) * sc;
            }
            const float v = o / lam;
            if constexpr (OUT_F32) reinterpret_cast<float*>(p.out)[out_row0 + e] = v;
            else reinterpret_cast<__nv_bfloat16*>(p.out)[out_row0 + e] = __float2bfloat16_rn(v);
          }
        }
      }
    }
    named_bar_sync(1, kConsumerWarps * 32);  // shared merge buffers free again
  };

  int it = 0;
  int split_idx = desc.z;
  for (int u = ub; u < ue; ++u, ++it) {
    if (seg_b < 0 || wk.t == 0) {
      if (seg_b >= 0) {
        finish_segment(seg_b, seg_g, split_idx);
        split_idx = 0;
      }
      seg_b = wk.b;
      seg_g = wk.g;
      L = p.ws.lens[seg_b];
      // query fragments (MMA B operand) of this kv head's G query heads
      const uint16_t* qbase = p.q + ((long long)seg_b * p.Hq + (long long)seg_g * p.G) * D;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int hh = nt * 8 + r;
        const bool valid = hh < p.G;
        const uint16_t* qrow = qbase + (long long)hh * D;
#pragma unroll
        for (int ks = 0; ks < C::kKSteps; ++ks) {
          if constexpr (!FP8) {
            qf[nt][ks][0] = valid ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * c) : 0u;
            qf[nt][ks][1] = valid ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 8 + 2 * c) : 0u;
          } else {
            // permuted k index: step ks covers d = 16 ks + 4c + {0,1} and {2,3}
            uint2 raw = valid ? *reinterpret_cast<const uint2*>(qrow + 16 * ks + 4 * c) : make_uint2(0, 0);
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

    const int s = it % C::kStages;
    const bool have = wait_bar(smem_u32(&full_bar[s]), (it / C::kStages) & 1, s_abort, status);
    const uint32_t kt = smem_u32(stages + s * C::kStageBytes);
    const uint32_t vt = kt + C::kTileBytes;
    float ksc = 1.f, vsc = 1.f;
    if constexpr (FP8) {
      ksc = info[s].k_scale;
      vsc = info[s].v_scale;
    }
    (void)have;

    // ---- S^T = K_w . Q^T
    float sacc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) sacc[nt][j] = 0.f;
    if constexpr (!FP8) {
#pragma unroll
      for (int ks = 0; ks < C::kKSteps; ++ks) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(tile_addr(kt, k_tok, 2 * ks + k_chk), a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_bf16(sacc[nt], a0, a1, a2, a3, qf[nt][ks][0], qf[nt][ks][1]);
      }
    } else {
#pragma unroll
      for (int kp = 0; kp < C::kKSteps / 2; ++kp) {
        uint32_t r0, r1, r2, r3;
        ldsm_x4(tile_addr(kt, k_tok, 2 * kp + k_chk), r0, r1, r2, r3);
        const uint32_t a[2][4] = {
            {e4m3x2_to_f16x2(r0 & 0xffff), e4m3x2_to_f16x2(r1 & 0xffff), e4m3x2_to_f16x2(r0 >> 16),
             e4m3x2_to_f16x2(r1 >> 16)},
            {e4m3x2_to_f16x2(r2 & 0xffff), e4m3x2_to_f16x2(r3 & 0xffff), e4m3x2_to_f16x2(r2 >> 16),
             e4m3x2_to_f16x2(r3 >> 16)}};
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            mma_f16(sacc[nt], a[h][0], a[h][1], a[h][2], a[h][3], qf[nt][2 * kp + h][0],
                    qf[nt][2 * kp + h][1]);
      }
    }

    // ---- online softmax (base 2)
    const int valid = L - (wk.t * kPageSize + tok0);  // live tokens in this warp's slice
    const float mul = p.scale_log2 * ksc;
    uint32_t pb[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float s0 = sacc[nt][0] * mul, s1 = sacc[nt][1] * mul;
      float s2 = sacc[nt][2] * mul, s3 = sacc[nt][3] * mul;
      if (r >= valid) { s0 = -INFINITY; s1 = -INFINITY; }
      if (r + 8 >= valid) { s2 = -INFINITY; s3 = -INFINITY; }
      float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 4));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 4));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 8));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 8));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 16));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 16));
      const float mn0 = fmaxf(m_run[nt][0], mx0), mn1 = fmaxf(m_run[nt][1], mx1);
      const float base0 = (mn0 == -INFINITY) ? 0.f : mn0;
      const float base1 = (mn1 == -INFINITY) ? 0.f : mn1;
      const float al0 = exp2f(m_run[nt][0] - base0), al1 = exp2f(m_run[nt][1] - base1);
      const float p0 = exp2f(s0 - base0), p2 = exp2f(s2 - base0);
      const float p1 = exp2f(s1 - base1), p3 = exp2f(s3 - base1);
      l_run[nt][0] = l_run[nt][0] * al0 + p0 + p2;
      l_run[nt][1] = l_run[nt][1] * al1 + p1 + p3;
      m_run[nt][0] = mn0;
      m_run[nt][1] = mn1;
#pragma unroll
      for (int i = 0; i < C::kMTiles; ++i) {
        acc[nt][i][0] *= al0;
        acc[nt][i][1] *= al1;
        acc[nt][i][2] *= al0;
        acc[nt][i][3] *= al1;
      }
      if constexpr (!FP8) {
        pb[nt][0] = movm_t(pack_bf16(p0, p1));
        pb[nt][1] = movm_t(pack_bf16(p2, p3));
      } else {
        pb[nt][0] = movm_t(pack_f16(p0 * vsc, p1 * vsc));
        pb[nt][1] = movm_t(pack_f16(p2 * vsc, p3 * vsc));
      }
    }

    // ---- O^T += V_w^T . P^T   (V rows past the length are zeroed in registers:
    // their probabilities are 0 but the slot may hold NaN/Inf garbage)
    const bool tail = valid < 16;
    const uint32_t m_lo = (2 * c < valid ? 0x0000ffffu : 0u) | (2 * c + 1 < valid ? 0xffff0000u : 0u);
    const uint32_t m_hi = (2 * c + 8 < valid ? 0x0000ffffu : 0u) | (2 * c + 9 < valid ? 0xffff0000u : 0u);
    uint32_t va[C::kMTiles][4];
    if constexpr (!FP8) {
#pragma unroll
      for (int i = 0; i < C::kMTiles; ++i)
        ldsm_x4_t(tile_addr(vt, v_tok, 2 * i + v_chk), va[i][0], va[i][1], va[i][2], va[i][3]);
    } else {
#pragma unroll
      for (int ip = 0; ip < C::kMTiles / 2; ++ip) {
        uint32_t r0, r1, r2, r3;
        ldsm_x4_t(tile_addr(vt, v_tok, 2 * ip + v_chk), r0, r1, r2, r3);
        // r0/r1: tokens [0,8)/[8,16) of chunk 2ip; r2/r3: same for chunk 2ip+1.
        // Each holds bytes {V(t,d), V(t,d+1), V(t+1,d), V(t+1,d+1)}.
        va[2 * ip][0] = e4m3x2_to_f16x2((uint16_t)__byte_perm(r0, 0, 0x0020));
        va[2 * ip][1] = e4m3x2_to_f16x2((uint16_t)__byte_perm(r0, 0, 0x0031));
        va[2 * ip][2] = e4m3x2_to_f16x2((uint16_t)__byte_perm(r1, 0, 0x0020));
        va[2 * ip][3] = e4m3x2_to_f16x2((uint16_t)__byte_perm(r1, 0, 0x0031));
        va[2 * ip + 1][0] = e4m3x2_to_f16x2((uint16_t)__byte_perm(r2, 0, 0x0020));
        va[2 * ip + 1][1] = e4m3x2_to_f16x2((uint16_t)__byte_perm(r2, 0, 0x0031));
        va[2 * ip + 1][2] = e4m3x2_to_f16x2((uint16_t)__byte_perm(r3, 0, 0x0020));
        va[2 * ip + 1][3] = e4m3x2_to_f16x2((uint16_t)__byte_perm(r3, 0, 0x0031));
      }
    }
    // all shared-memory reads of this stage are done: hand it back
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&empty_bar[s]));
    if (tail) {
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
      for (int nt = 0; nt < NT; ++nt) {
        if constexpr (!FP8) mma_bf16(acc[nt][i], va[i][0], va[i][1], va[i][2], va[i][3], pb[nt][0], pb[nt][1]);
        else mma_f16(acc[nt][i], va[i][0], va[i][1], va[i][2], va[i][3], pb[nt][0], pb[nt][1]);
      }

    if (u + 1 < ue) wk.next(ts, p.Hkv);
  }
  if (seg_b >= 0) finish_segment(seg_b, seg_g, split_idx);
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
bool make_cache_map(CUtensorMap* tm, const void* base, int num_pages, int Hkv, int D, bool fp8) {
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

template <int D, int NT, bool FP8, bool OUT_F32>
hpa_status launch(const CUtensorMap& tk, const CUtensorMap& tv, const RunParams& p, int grid,
                  cudaStream_t stream) {
  using C = Cfg<D, NT, FP8>;
  auto kern = decode_kernel<D, NT, FP8, OUT_F32>;
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

template <int D, bool FP8, bool OUT_F32>
hpa_status launch_nt(int nt, const CUtensorMap& tk, const CUtensorMap& tv, const RunParams& p,
                     int grid, cudaStream_t s) {
  return nt == 1 ? launch<D, 1, FP8, OUT_F32>(tk, tv, p, grid, s)
                 : launch<D, 2, FP8, OUT_F32>(tk, tv, p, grid, s);
}

}  // namespace
}  // namespace hpa

using namespace hpa;

extern "C" hpa_status hpa_decode_run(const void* q, const void* k_cache, const void* v_cache,
                                     const float* k_scale, const float* v_scale,
                                     hpa_kv_dtype kv_dtype, const int32_t* page_table,
                                     int pt_stride, int num_pages, void* out,
                                     hpa_out_dtype out_dtype, int batch, int num_q_heads,
                                     int num_kv_heads, int head_dim, float softmax_scale,
                                     int grid, void* workspace, size_t ws_bytes, void* stream) {
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
  if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return HPA_ERR_UNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return HPA_ERR_UNSUPPORTED;
  if (fp8 && head_dim != 128) return HPA_ERR_UNSUPPORTED;
  if ((long long)num_pages * num_kv_heads * kPageSize > 0x7fffffffLL) return HPA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache)) & 15)
    return HPA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q) & 7) || (reinterpret_cast<uintptr_t>(out) & 3))
    return HPA_ERR_INVALID_ARG;
  WsLayout L;
  if (!ws_layout(batch, num_kv_heads, num_q_heads, head_dim, grid, &L)) return HPA_ERR_INVALID_ARG;
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
  p.B = batch;
  p.Hq = num_q_heads;
  p.Hkv = num_kv_heads;
  p.G = G;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.ws = ws_view(workspace, L);
  p.grid = grid;
  const int nt = G > 8 ? 2 : 1;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool f32 = out_dtype == HPA_OUT_F32;
  if (fp8)
    return f32 ? launch_nt<128, true, true>(nt, tk, tv, p, grid, s)
               : launch_nt<128, true, false>(nt, tk, tv, p, grid, s);
  if (head_dim == 128)
    return f32 ? launch_nt<128, false, true>(nt, tk, tv, p, grid, s)
               : launch_nt<128, false, false>(nt, tk, tv, p, grid, s);
  return f32 ? launch_nt<64, false, true>(nt, tk, tv, p, grid, s)
             : launch_nt<64, false, false>(nt, tk, tv, p, grid, s);
}
