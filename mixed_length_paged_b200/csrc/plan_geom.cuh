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

// Largest i in [0, n) with key(i) <= T, for key non-decreasing and key(0) <=
// T, found by a whole warp (all 32 lanes call it with the same arguments):
// each round probes 32 evenly spaced candidates at once and keeps the gap
// after the last one that passes, so n <= 1024 takes two rounds.
template <class Key>
__device__ __forceinline__ int warp_last_le(int n, long long T, Key key, int lane) {
  int lo = 0, len = n;
  while (len > 1) {
    const int step = (len + 31) >> 5;
    const bool ok = lane * step < len && key(lo + lane * step) <= T;
    const int k = 31 - __clz(__ballot_sync(0xffffffffu, ok));  // lane 0 always passes
    lo += k * step;
    len = min(step, len - k * step);
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

// Per-sequence prefix data of one step's lengths: tile offsets ts[0..B], and
// which sequences hold tiles (bit b % 32 of word b / 32) with the count of
// such sequences before each group of 32 (nzp[0..ceil(B/32)]).
struct SeqIdx {
  const int32_t* ts;
  const uint32_t* nzm;
  const int32_t* nzp;
  int B, Hkv;
  // sequences with tiles among [0, b), 0 <= b <= B
  __device__ __forceinline__ int nz(int b) const {
    const int w = b >> 5, r = b & 31;
    return nzp[w] + (r ? __popc(nzm[w] & ((1u << r) - 1u)) : 0);
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
//
// The primary ranges split the primary units' COST evenly: every unit costs
// q and the last unit of each segment e more (a segment end: the state
// hand-off and combine).  With K(x) the cost of units [0, x), primary range c
// starts at x_c, the largest x <= U1 with P K(x) <= c K(U1), i.e. K(x) <=
// floor(c K1 / P) with K1 = K(U1); unit u < U1 lies in range floor((K(u+1) P
// - 1) / K1).  With e = 0 (any q) this is the even partition above; then K(x)
// is taken as x, so no sequence lookups are made.  The weights apply only if
// K1 >= (q + e) P: then consecutive cut targets differ by at least the
// largest unit cost, so every primary range holds a unit (as in the even
// partition, where U1 >= P) and the ranges holding a segment are consecutive,
// which the partial slots need.  Otherwise the units are split evenly.
struct DynGeom {
  long long U, P, Pd, U1, Ut, M, K1;
  int q, e;
  bool cost;  // e > 0, U > P and K1 >= (q + e) P: the primary cuts are by cost
  SeqIdx si;
  FloorDiv by_Pd, by_M, by_K1, by_Ut;
  // (called by whole warps, all lanes with the same arguments)
  __device__ void init(long long units, long long ctas, int tail_den, int tail_chunks,
                       int tail_min, int unit_cost, int end_cost, const SeqIdx& idx, int lane) {
    U = units;
    P = ctas;
    si = idx;
    q = unit_cost;
    e = end_cost;
    if (U <= P) {
      Pd = U; U1 = U; Ut = 0; M = 0;
    } else {
      Pd = P;
      const bool tail = tail_den > 0 && U >= (long long)tail_min * P;
      Ut = tail ? std::min<long long>(U / tail_den, U - P) : 0;
      U1 = U - Ut;
      M = std::min<long long>((long long)tail_chunks * P, Ut);
    }
    cost = e > 0 && U > P;
    if (cost) {
      K1 = K_warp(U1, lane);
      cost = K1 >= (long long)(q + e) * P;
    }
    if (!cost) K1 = U1;
  }
  // cost of the units before sequence b's first unit
  __device__ __forceinline__ long long Kseq(int b) const {
    return ((long long)q * si.ts[b] + (long long)e * si.nz(b)) * si.Hkv;
  }
  // K(x): cost of units [0, x), 0 <= x <= U (x itself without cost weights)
  __device__ __forceinline__ long long K(long long x) const {
    if (!cost) return x;
    if (x >= U) return Kseq(si.B);
    return K_search(x);
  }
  // K(x) for x < U under cost weights, by one thread (K_search) or a warp
  __device__ __forceinline__ long long K_search(long long x) const {
    return K_in(seq_of_unit(si.ts, si.B, si.Hkv, x), x);
  }
  __device__ __forceinline__ long long K_warp(long long x, int lane) const {
    if (x >= U) return Kseq(si.B);
    const int32_t* ts = si.ts;
    const int Hkv = si.Hkv;
    return K_in(warp_last_le(si.B, x, [&](int i) { return (long long)ts[i] * Hkv; }, lane), x);
  }
  // K(x) for unit x < U of sequence b
  __device__ __forceinline__ long long K_in(int b, long long x) const {
    const int n = si.ts[b + 1] - si.ts[b];
    const int rem = (int)(x - (long long)si.ts[b] * si.Hkv);  // < Hkv n <= U < 2^31
    const int g = rem / n;
    return Kseq(b) + (long long)g * ((long long)q * n + e) + (long long)q * (rem - g * n);
  }
  // Sequence, kv head, tile and tile count (b, g, t, n) of the largest x <=
  // U1 with K(x) <= T, under cost weights and for T < K1; x = ts[b] Hkv + g n
  // + t.
  __device__ __forceinline__ int4 xinv_pos(long long T) const {
    int lo = 0, hi = si.B - 1;  // largest b with Kseq(b) <= T (Kseq(0) = 0)
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (Kseq(mid) <= T) lo = mid; else hi = mid - 1;
    }
    return xinv_in(lo, T);
  }
  // the same, found by a whole warp
  __device__ __forceinline__ int4 xinv_pos_warp(long long T, int lane) const {
    return xinv_in(warp_last_le(si.B, T, [&](int i) { return Kseq(i); }, lane), T);
  }
  // ... given lo, the last sequence with Kseq(lo) <= T
  __device__ __forceinline__ int4 xinv_in(int lo, long long T) const {
    // T < K1 <= K(U): sequence lo has tiles and y < Hkv (q n + e)
    const int n = si.ts[lo + 1] - si.ts[lo];
    const long long sc = (long long)q * n + e;  // one segment of this sequence
    const long long y = T - Kseq(lo);
    long long g, r;
    if (((unsigned long long)y | (unsigned long long)sc) >> 32) {
      g = y / sc;
      r = (y - g * sc) / q;
    } else {  // (the usual case: 32-bit divisions)
      g = (unsigned)y / (unsigned)sc;
      r = ((unsigned)y - (unsigned)g * (unsigned)sc) / (unsigned)q;
    }
    const long long j = std::min(r, (long long)n - 1);
    return make_int4(lo, (int)g, (int)j, n);
  }
  __device__ __forceinline__ long long unit_at(int4 pos) const {
    return (long long)si.ts[pos.x] * si.Hkv + (long long)pos.y * pos.w + pos.z;
  }
  // largest x <= U1 with K(x) <= T (xinv_warp: by a whole warp)
  __device__ __forceinline__ long long xinv(long long T) const {
    if (!cost) return std::min(T, U1);
    if (T >= K1) return U1;
    return unit_at(xinv_pos(T));
  }
  __device__ __forceinline__ long long xinv_warp(long long T, int lane) const {
    if (!cost) return std::min(T, U1);
    if (T >= K1) return U1;
    return unit_at(xinv_pos_warp(T, lane));
  }
  // the divisors whose reciprocals init_div takes, in order
  __device__ long long divisor(int i) const { return i == 0 ? Pd : i == 1 ? M : i == 2 ? K1 : Ut; }
  __device__ void init_div(const double* r) {
    by_Pd.init(Pd, r[0]);
    by_M.init(M, r[1]);
    by_K1.init(K1, r[2]);
    by_Ut.init(Ut, r[3]);
  }
  __device__ long long ranges() const { return P + M; }
  // range holding unit u, given Ku1 = K(u + 1) (used only if u < U1)
  __device__ long long range_of_k(long long u, long long Ku1) const {
    return u < U1 ? by_K1(Ku1 * Pd - 1) : P + by_Ut((u - U1 + 1) * M - 1);
  }
  __device__ long long range_of(long long u) const {
    return range_of_k(u, u < U1 ? K(u + 1) : 0);
  }
  __device__ void bounds(long long c, long long* ub, long long* ue) const {
    if (c < P) {
      if (c < Pd) {
        *ub = xinv(by_Pd(c * K1));
        *ue = xinv(by_Pd((c + 1) * K1));
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
// plan, from the tile offsets ts[0..B].  lane >= 0: called by a whole warp,
// all lanes with the same c, which then searches with the warp.
__device__ __forceinline__ void dyn_range_desc(const DynGeom& dg, const int32_t* ts, int B, int Hkv,
                                               long long c, int4* d0, int4* d1, int lane = -1) {
  long long ub, ue;
  int b0 = 0, g0 = 0, t0 = 0, n0 = 0;
  if (dg.cost && c < dg.P) {
    // (primary ranges under cost weights are never empty and start below U1)
    const long long Tb = dg.by_Pd(c * dg.K1), Te = dg.by_Pd((c + 1) * dg.K1);
    const int4 pos = lane >= 0 ? dg.xinv_pos_warp(Tb, lane) : dg.xinv_pos(Tb);
    b0 = pos.x;
    g0 = pos.y;
    t0 = pos.z;
    n0 = pos.w;
    ub = dg.unit_at(pos);
    ue = lane >= 0 ? dg.xinv_warp(Te, lane) : dg.xinv(Te);
  } else {
    dg.bounds(c, &ub, &ue);
    if (ub < ue) {
      b0 = seq_of_unit(ts, B, Hkv, ub);
      n0 = ts[b0 + 1] - ts[b0];
      const int rem = (int)(ub - (long long)ts[b0] * Hkv);  // < Hkv * n0 < 2^31
      g0 = rem / n0;
      t0 = rem - g0 * n0;
    }
  }
  *d0 = make_int4((int)ub, (int)ue, b0, g0);
  *d1 = make_int4(t0, n0, 0, 0);
}

// Segment descriptor (first partial slot or -1, ranges holding it) of segment
// s of the dynamic plan.
// The costs it needs are closed forms in (b, g): K(segment start) = Kseq(b)
// + g (q n + e), each tile q more, the segment's last e more still.  The
// segment's first piece opens its range iff the unit before the segment lies
// in an earlier range: every primary range and tail chunk holds a unit when
// U > P, and for U <= P range c is unit c.
__device__ __forceinline__ int2 dyn_seg_desc(const DynGeom& dg, const int32_t* ts, int Hkv, int s) {
  const int b = s / Hkv, g = s - b * Hkv;
  const long long n = ts[b + 1] - ts[b];
  int nsplit = 0, slot0 = -1;
  if (n > 0) {
    const long long seg_start = (long long)ts[b] * Hkv + (long long)g * n;
    long long k0 = seg_start, k1 = seg_start + 1, kn = seg_start + n;  // K at start, +1, end
    if (dg.cost) {
      const long long sc = (long long)dg.q * n + dg.e;
      k0 = dg.Kseq(b) + g * sc;
      k1 = k0 + dg.q + (n == 1 ? dg.e : 0);
      kn = k0 + sc;
    }
    const long long r0 = dg.range_of_k(seg_start, k1);
    nsplit = (int)(dg.range_of_k(seg_start + n - 1, kn) - r0 + 1);
    if (nsplit > 1) {
      const bool opens = seg_start == 0 || dg.range_of_k(seg_start - 1, k0) != r0;
      slot0 = (int)(2 * r0 + (opens ? 0 : 1));
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
