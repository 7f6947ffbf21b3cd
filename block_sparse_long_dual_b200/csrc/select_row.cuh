// Warp-level selection of one row's key blocks ("Prism: Spectral-Aware
// Block-Sparse Attention" §1: attention runs over a chosen subset of blocks),
// shared by the standalone selection kernel and the fused score+select kernel.
//
// The row's probabilities sit in registers (lane l holds blocks l, l + 32,
// l + 64, ...).  Probabilities are >= 0, so their float32 bit patterns order
// like the values; candidates carry their bit pattern as a signed key and
// non-candidates (forced blocks, j > i) key -1.  The kept candidates are a
// prefix of the order (probability desc, index asc): {key > T} plus the
// lowest-index entries of {key == T} for one threshold key T, found by
// bisection over the 31-bit key range:
//   top-k:  T = the largest key with #{key >= T} >= k; take k - #{key > T} ties.
//   mass:   T = the smallest key with forced + sum_{key > T} p < mass (float64
//           sums), i.e. the value of the last candidate added; ties are added in
//           index order while the running sum stays below mass.
// The kept set (forced blocks included) is written ascending, padded with -1.
// Once the keys that can still matter (top-k: key >= lo; mass: key > lo, lo
// the bisection's lower bracket) number at most 64, they are compacted into
// shared memory, two per lane, and the remaining bisection steps scan those
// instead of every register slot.
#pragma once

#include "common.cuh"

namespace sfa {

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// prob(j) returns the float32 probability of block j (called for j <= i only).
// Writes out[0 .. kmax) and returns the kept count.  All 32 lanes must call it.
template <int NPL, typename ProbFn>
__device__ int select_row_warp(ProbFn prob, int i, int k, double mass, unsigned flags, int* out, int kmax) {
  const int lane = threadIdx.x & 31;
  const int f1 = ((flags & SFA_KEEP_SINK) && i > 0) ? 0 : -1;
  const int nforced = f1 >= 0 ? 2 : 1;
  const int nc = i + 1 - nforced;
  const int tmax = i / 32 + 1;  // register slots that hold blocks <= i

  int key[NPL];  // candidate: bit pattern of its probability (the value is __uint_as_float(key))
#pragma unroll
  for (int t = 0; t < NPL; ++t) {
    const int j = t * 32 + lane;
    int kk = -1;
    if (t < tmax && j <= i && j != i && j != f1) kk = (int)__float_as_uint(prob(j));
    key[t] = kk;
  }

  // Compaction buffer: 64 keys per warp (the kernels that call this run 8 warps per CTA).
  __shared__ int ckeys[8][64];
  int* cb = ckeys[(threadIdx.x >> 5) & 7];
  // Copies the keys with key >= lo0 (in register-slot order) into cb, padding with -1, and returns
  // this lane's two of them (slots lane and lane + 32).
  auto compact = [&](int lo0, int& k0, int& k1) {
    int base = 0;
    const unsigned lt2 = (1u << lane) - 1u;
#pragma unroll
    for (int t = 0; t < NPL; ++t) {
      const bool in = t < tmax && key[t] >= lo0;
      const unsigned bm = __ballot_sync(0xffffffffu, in);
      if (in) cb[base + __popc(bm & lt2)] = key[t];
      base += __popc(bm);
    }
    __syncwarp();
    k0 = lane < base ? cb[lane] : -1;
    k1 = lane + 32 < base ? cb[lane + 32] : -1;
    __syncwarp();
  };

  int T = -1;         // threshold key; candidates with key > T are kept
  int take_ties = 0;  // number of key == T candidates kept, lowest index first
  if (k >= 0) {
    if (k >= nc) {
      T = -1;  // every candidate
    } else if (k > 0) {
      int lo = 0, hi = 0x7F800001;  // #{key >= lo} >= k, #{key >= hi} < k
      int clo = nc;                 // #{key >= lo}
      while (hi - lo > 1 && clo > 64) {
        const int mid = lo + ((hi - lo) >> 1);
        int c = 0;
#pragma unroll
        for (int t = 0; t < NPL; ++t) c += (t < tmax && key[t] >= mid) ? 1 : 0;
        c = __reduce_add_sync(0xffffffffu, c);
        if (c >= k) { lo = mid; clo = c; } else { hi = mid; }
      }
      int g = 0;
      if (hi - lo > 1) {
        // Every key >= lo is in the compacted set, so counts at mid >= lo are unchanged.
        int k0, k1;
        compact(lo, k0, k1);
        while (hi - lo > 1) {
          const int mid = lo + ((hi - lo) >> 1);
          const int c = __reduce_add_sync(0xffffffffu, (k0 >= mid ? 1 : 0) + (k1 >= mid ? 1 : 0));
          if (c >= k) lo = mid; else hi = mid;
        }
        g = __reduce_add_sync(0xffffffffu, (k0 > lo ? 1 : 0) + (k1 > lo ? 1 : 0));
      } else {
#pragma unroll
        for (int t = 0; t < NPL; ++t) g += (t < tmax && key[t] > lo) ? 1 : 0;
        g = __reduce_add_sync(0xffffffffu, g);
      }
      T = lo;
      take_ties = k - g;
    } else {
      T = 0x7F800001;  // k = 0: no candidate
    }
  } else {
    // Running sum starts with the forced blocks.
    const double cum_forced = (double)prob(i) + (f1 >= 0 ? (double)prob(f1) : 0.0);
    double all = 0.0;
#pragma unroll
    for (int t = 0; t < NPL; ++t)
      all += (t < tmax && key[t] >= 0) ? (double)__uint_as_float((unsigned)key[t]) : 0.0;
    all = warp_sum_f64(all);
    if (cum_forced >= mass) {
      T = 0x7F800001;  // nothing added
    } else if (cum_forced + all < mass) {
      T = -1;  // every candidate added
    } else {
      int lo = -1, hi = 0x7F800000;  // F(lo) >= mass, F(hi) < mass, F(U) = forced + sum_{key > U} p
      int cgt = nc;                  // #{key > lo}
      while (hi - lo > 1 && cgt > 64) {
        const int mid = lo + ((hi - lo) >> 1);
        double sacc = 0.0;
        int c = 0;
#pragma unroll
        for (int t = 0; t < NPL; ++t) {
          const bool gt = t < tmax && key[t] > mid;
          sacc += gt ? (double)__uint_as_float((unsigned)key[t]) : 0.0;
          c += gt ? 1 : 0;
        }
        sacc = warp_sum_f64(sacc);
        c = __reduce_add_sync(0xffffffffu, c);
        if (cum_forced + sacc < mass) { hi = mid; } else { lo = mid; cgt = c; }
      }
      // From here on only keys > lo can change F or the ties at hi: every one of them is in the
      // compacted set when the loop above stopped on the count.
      double sg = 0.0;
      int e = 0;
      if (cgt <= 64) {
        int k0, k1;
        compact(lo + 1, k0, k1);
        auto val = [](int kk) { return kk >= 0 ? (double)__uint_as_float((unsigned)kk) : 0.0; };
        while (hi - lo > 1) {
          const int mid = lo + ((hi - lo) >> 1);
          const double sacc = warp_sum_f64((k0 > mid ? val(k0) : 0.0) + (k1 > mid ? val(k1) : 0.0));
          if (cum_forced + sacc < mass) hi = mid; else lo = mid;
        }
        sg = (k0 > hi ? val(k0) : 0.0) + (k1 > hi ? val(k1) : 0.0);
        e = (k0 == hi ? 1 : 0) + (k1 == hi ? 1 : 0);
      } else {
#pragma unroll
        for (int t = 0; t < NPL; ++t) {
          if (t < tmax && key[t] > hi) sg += (double)__uint_as_float((unsigned)key[t]);
          if (t < tmax && key[t] == hi) ++e;
        }
      }
      // hi is the key of the last candidate added; add its ties in index order while below mass.
      sg = cum_forced + warp_sum_f64(sg);
      e = __reduce_add_sync(0xffffffffu, e);
      const double tv = (double)__uint_as_float((unsigned)hi);
      int r = 0;
      double run = sg;
      while (r < e && run < mass) {
        run += tv;
        ++r;
      }
      T = hi;
      take_ties = r;
    }
  }

  // Ascending compaction of forced + kept candidates.
  int pos = 0, ties = 0;
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int t = 0; t < NPL; ++t) {
    if (t < tmax) {
      const int j = t * 32 + lane;
      const bool tie = key[t] >= 0 && key[t] == T;
      const unsigned tb = __ballot_sync(0xffffffffu, tie);
      const bool keep_tie = tie && (ties + __popc(tb & lt)) < take_ties;
      const bool keep = (j <= i) && (j == i || j == f1 || key[t] > T || keep_tie);
      const unsigned kb = __ballot_sync(0xffffffffu, keep);
      if (keep) out[pos + __popc(kb & lt)] = j;
      pos += __popc(kb);
      ties += __popc(tb);
    }
  }
  for (int q = pos + lane; q < kmax; q += 32) out[q] = -1;
  return pos;
}

}  // namespace sfa
