// prologue_math.cuh -- the per-row arithmetic of the decode prologue
// (bitbyai.com "vLLM x HPC-Ops", Attention Backend: RoPE, query-key
// normalisation and the KV write fused into one prologue), shared by the
// standalone prologue kernel and the decode kernel's fused prologue so that
// both produce the same bits.
//
// One warp handles one head row of D elements.  Lane l owns the rotary pairs
// (i, i + D/2) for i = l + 32 j, j < D/64, so RMSNorm's sum of squares is one
// warp reduction and the rotate-half RoPE needs no data exchange.
//
// Precision: RMSNorm and the rotation run in fp32.  The rotation angle
// pos * theta^(-2i/D) is formed and reduced modulo 2*pi in fp64 before the
// fp32 sine/cosine: at pos ~ 65536 an fp32 angle would already be off by
// ~4e-3 rad.
#pragma once

#include <cuda_bf16.h>

namespace hpa {

template <int D>
struct RopeLane {
  static constexpr int kPairs = D / 64;  // rotary pairs per lane
  float cs[kPairs], sn[kPairs];

  // cos/sin of this lane's angles at position pos
  __device__ __forceinline__ void init(int pos, int lane, double log2_theta) {
#pragma unroll
    for (int j = 0; j < kPairs; ++j) {
      const int i = lane + 32 * j;
      const double w = exp2(-(2.0 * i / D) * log2_theta);  // theta^(-2i/D)
      double phi = (double)pos * w;
      const double two_pi = 6.283185307179586476925;
      phi = fma(-two_pi, rint(phi / two_pi), phi);
      sincosf((float)phi, &sn[j], &cs[j]);
    }
  }
};

// RMSNorm(src; gamma, eps) then RoPE, rounded to bf16, for one row; the whole
// warp calls it and lane l gets the results for elements i = l + 32 j (lo[j])
// and i + D/2 (hi[j]).  Every rounding step is spelled out (fma, __fmul_rn,
// ...), so the bits do not depend on how the compiler would contract the
// expressions in the kernel this is inlined into.
template <int D>
__device__ __forceinline__ void norm_rope_vals(const __nv_bfloat16* src, const float* gamma,
                                               float eps, const RopeLane<D>& r, int lane,
                                               __nv_bfloat16 (&lo)[D / 64],
                                               __nv_bfloat16 (&hi)[D / 64]) {
  constexpr int kPairs = RopeLane<D>::kPairs;
  float x[2 * kPairs];  // x[j] = element lane+32j (first half), x[kPairs+j] = its partner
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < kPairs; ++j) {
    x[j] = __bfloat162float(src[lane + 32 * j]);
    x[kPairs + j] = __bfloat162float(src[lane + 32 * j + D / 2]);
    ss = fmaf(x[j], x[j], ss);
    ss = fmaf(x[kPairs + j], x[kPairs + j], ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float rinv = __frcp_rn(__fsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)D), eps)));
#pragma unroll
  for (int j = 0; j < kPairs; ++j) {
    const int i = lane + 32 * j;
    const float a = __fmul_rn(__fmul_rn(x[j], rinv), gamma[i]);
    const float c2 = __fmul_rn(__fmul_rn(x[kPairs + j], rinv), gamma[i + D / 2]);
    lo[j] = __float2bfloat16_rn(fmaf(a, r.cs[j], -__fmul_rn(c2, r.sn[j])));
    hi[j] = __float2bfloat16_rn(fmaf(c2, r.cs[j], __fmul_rn(a, r.sn[j])));
  }
}

// norm_rope_vals stored to a plain row dst (which may alias src: each lane
// reads its elements before writing them), and to dst2 if not null.  With
// dst == nullptr nothing is stored (dst2 is ignored too).
template <int D>
__device__ __forceinline__ void norm_rope_row(const __nv_bfloat16* src, __nv_bfloat16* dst,
                                              __nv_bfloat16* dst2, const float* gamma, float eps,
                                              const RopeLane<D>& r, int lane) {
  constexpr int kPairs = RopeLane<D>::kPairs;
  if (!dst) return;  // warp-uniform: the whole warp skips the row
  __nv_bfloat16 lo[kPairs], hi[kPairs];
  norm_rope_vals<D>(src, gamma, eps, r, lane, lo, hi);
#pragma unroll
  for (int j = 0; j < kPairs; ++j) {
    const int i = lane + 32 * j;
    dst[i] = lo[j];
    dst[i + D / 2] = hi[j];
    if (dst2) {
      dst2[i] = lo[j];
      dst2[i + D / 2] = hi[j];
    }
  }
}

}  // namespace hpa
