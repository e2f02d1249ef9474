// plan_geom.cuh -- the dynamic plan's closed-form geometry, shared by the
// plan kernel and the decode kernel's in-kernel planning (hpa_decode_step),
// so that both cut the unit list into exactly the same ranges.
#pragma once

#include <algorithm>

#include "hpa_common.cuh"

namespace hpa {

// Largest b in [0, B) with tile_start[b] * Hkv <= u (u < U).
__device__ __forceinline__ int seq_of_unit(const int32_t* tile_start, int B, int Hkv, long long u) {
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
// the P primary ranges and the last Ut units over M tail chunks, handed out at
// run time to whichever CTA is free, where for the tail parameters (den, k,
// mn) Ut = min(floor(U/den), U - P) if den > 0 and U >= mn P, else 0, and M =
// min(kP, Ut).  The parameters are the library's tuning (HPA_TAIL_*_DEFAULT
// unless the caller gives others); no tail is the plain even partition of
// all U units over the P CTAs.  For n units spread
// over m ranges as [floor(cn/m), floor((c+1)n/m)), the range holding unit u is
// the largest c with floor(cn/m) <= u, i.e. floor(((u+1)m - 1) / n).
struct DynGeom {
  long long U, P, Pd, U1, Ut, M;
  FloorDiv by_Pd, by_M, by_U1, by_Ut;
  __device__ void init(long long units, long long ctas, int tail_den, int tail_chunks,
                       int tail_min) {
    U = units;
    P = ctas;
    if (U <= P) {
      Pd = U; U1 = U; Ut = 0; M = 0;
    } else {
      Pd = P;
      const bool tail = tail_den > 0 && U >= (long long)tail_min * P;
      Ut = tail ? std::min<long long>(U / tail_den, U - P) : 0;
      U1 = U - Ut;
      M = std::min<long long>((long long)tail_chunks * P, Ut);
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


// The dynamic plan's shape for U units over P persistent CTAs; r receives the
// reciprocals init_div takes (one thread per divisor, or all four in one).
__device__ __forceinline__ void dyn_reciprocals(const DynGeom& dg, double* r) {
  for (int i = 0; i < 4; ++i) {
    const long long d = dg.divisor(i);
    r[i] = d > 0 ? 1.0 / (double)d : 0.0;
  }
}

// Unit range and first-unit state (b0, g0, t0, n0) of range c of the dynamic
// plan, from the tile offsets ts[0..B].
__device__ __forceinline__ void dyn_range_desc(const DynGeom& dg, const int32_t* ts, int B, int Hkv,
                                               long long c, int4* d0, int4* d1) {
  long long ub, ue;
  int b0 = 0, g0 = 0, t0 = 0, n0 = 0;
  dg.bounds(c, &ub, &ue);
  if (ub < ue) {
    b0 = seq_of_unit(ts, B, Hkv, ub);
    n0 = ts[b0 + 1] - ts[b0];
    const int rem = (int)(ub - (long long)ts[b0] * Hkv);  // < Hkv * n0 < 2^31
    g0 = rem / n0;
    t0 = rem - g0 * n0;
  }
  *d0 = make_int4((int)ub, (int)ue, b0, g0);
  *d1 = make_int4(t0, n0, 0, 0);
}

// Segment descriptor (first partial slot or -1, ranges holding it) of segment
// s of the dynamic plan.
__device__ __forceinline__ int2 dyn_seg_desc(const DynGeom& dg, const int32_t* ts, int Hkv, int s) {
  const int b = s / Hkv, g = s - b * Hkv;
  const long long n = ts[b + 1] - ts[b];
  int nsplit = 0, slot0 = -1;
  if (n > 0) {
    const long long seg_start = (long long)ts[b] * Hkv + (long long)g * n;
    const long long r0 = dg.range_of(seg_start);
    nsplit = (int)(dg.range_of(seg_start + n - 1) - r0 + 1);
    if (nsplit > 1) {
      long long ub, ue;
      dg.bounds(r0, &ub, &ue);
      slot0 = (int)(2 * r0 + (ub == seg_start ? 0 : 1));
    }
  }
  return make_int2(slot0, nsplit);
}

// LENGTH_AWARE plan geometry (bitbyai.com "vLLM x HPC-Ops", Attention
// Backend: short requests are finished first, long ones spread over the
// grid): the dynamic partition with every cut point x moved by snap().  If x
// lies strictly inside a segment [s0, s0 + n), a = x - s0: when a < m or
// n - a < m it moves to the nearer end of the segment (s0 on a tie), else it
// stays.  A segment of fewer than 2m tiles stays whole, and the first and
// last pieces of a cut segment have at least m tiles.  snap() is
// non-decreasing in x and moves a cut by less than m, so the ranges stay
// contiguous and in order, and the range holding unit u is found among the
// dynamic ranges within m - 1 units of u.
struct LaGeom {
  const DynGeom* dg;
  const int32_t* ts;
  int B, Hkv;
  long long m;

  __device__ long long snap(long long x) const {
    if (m <= 1 || x <= 0 || x >= dg->U) return x;
    const int b = seq_of_unit(ts, B, Hkv, x);
    const long long n = ts[b + 1] - ts[b];
    const long long base = (long long)ts[b] * Hkv;
    const long long a = (x - base) % n;  // tiles of x's segment before x
    if (a == 0) return x;
    const long long r = n - a;
    if (a < m || r < m) return a <= r ? x - a : x + r;
    return x;
  }
  // first unit of range c (c = V: U), before and after the move
  __device__ long long raw_start(long long c) const {
    if (c >= dg->ranges()) return dg->U;
    long long ub, ue;
    dg->bounds(c, &ub, &ue);
    return ub;
  }
  __device__ void bounds(long long c, long long* ub, long long* ue) const {
    long long a, e;
    dg->bounds(c, &a, &e);
    *ub = snap(a);
    *ue = snap(e);
  }
  // the last range whose moved start is <= u (for u < U: the range holding u)
  __device__ long long range_of(long long u) const {
    long long lo = dg->range_of(u - (m - 1) > 0 ? u - (m - 1) : 0);
    long long hi = dg->range_of(u + (m - 1) < dg->U - 1 ? u + (m - 1) : dg->U - 1);
    while (lo < hi) {
      const long long mid = (lo + hi + 1) >> 1;
      if (snap(raw_start(mid)) <= u) lo = mid; else hi = mid - 1;
    }
    return lo;
  }
};

// Range descriptor (as dyn_range_desc) of range c of the length-aware plan.
__device__ __forceinline__ void la_range_desc(const LaGeom& lg, long long c, int4* d0, int4* d1) {
  long long ub, ue;
  int b0 = 0, g0 = 0, t0 = 0, n0 = 0;
  lg.bounds(c, &ub, &ue);
  if (ub < ue) {
    b0 = seq_of_unit(lg.ts, lg.B, lg.Hkv, ub);
    n0 = lg.ts[b0 + 1] - lg.ts[b0];
    const int rem = (int)(ub - (long long)lg.ts[b0] * lg.Hkv);
    g0 = rem / n0;
    t0 = rem - g0 * n0;
  }
  *d0 = make_int4((int)ub, (int)ue, b0, g0);
  *d1 = make_int4(t0, n0, 0, 0);
}

// Segment descriptor (as dyn_seg_desc) of segment s of the length-aware plan.
// The ranges holding a segment are consecutive, as the merge's slot order
// needs: the cuts inside a segment did not move, so they are distinct, and
// only a segment's ends can collect several cuts (empty ranges).
__device__ __forceinline__ int2 la_seg_desc(const LaGeom& lg, int s) {
  const int b = s / lg.Hkv, g = s - b * lg.Hkv;
  const long long n = lg.ts[b + 1] - lg.ts[b];
  int nsplit = 0, slot0 = -1;
  if (n > 0) {
    const long long seg_start = (long long)lg.ts[b] * lg.Hkv + (long long)g * n;
    const long long r0 = lg.range_of(seg_start);
    nsplit = (int)(lg.range_of(seg_start + n - 1) - r0 + 1);
    if (nsplit > 1) {
      long long ub, ue;
      lg.bounds(r0, &ub, &ue);
      slot0 = (int)(2 * r0 + (ub == seg_start ? 0 : 1));
    }
  }
  return make_int2(slot0, nsplit);
}

}  // namespace hpa
