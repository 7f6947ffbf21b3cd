// Block logits and the causal block softmax on the int8 tensor cores, for the
// estimate of "Prism: Spectral-Aware Block-Sparse Attention" (§3.1 dual-band
// pooling with §3.2's per-band temperature, §5: the estimate is made of
// block-level matrix products only).  Serves head dim 128 and the plain
// calibrated logit (every flag except the per-band-softmax and per-block
// temperature readings, which keep the float64 kernel of scores.cu).
//
// The logit s_ij = sum_d qt_id kbar_jd, qt = qbar / (tau^band(d) sqrt(d)), is
// taken exactly enough for a float64 softmax through integer products:
//   score_slices  per row x of qt (query blocks) or kbar (key blocks), a power
//                 of two 2^e with |x 2^e| < 1/2, and five signed digits d_a in
//                 [-64, 64]: x 2^e = sum_a d_a 2^-7(a+1) + r, |r| <= 2^-36.
//   score_i8      CTA per (b, h, tile of 128 query blocks).  For 48 key blocks
//                 at a time, the 15 digit pairs (a, b) with a + b <= 4 go to
//                 the tensor core (kind::i8, M = 128, N = 48, K = 32 steps over
//                 the 128 dims), grouped by level a + b into five int32
//                 accumulators in TMEM (exact: |sum| <= 5 * 128 * 64^2 < 2^31);
//                 the epilogue combines them in float64,
//                   s_ij = 2^(-e_i - f_j - 14) sum_s A_s 2^(-7 s),
//                 and the dropped pairs and the digits' remainders leave an
//                 error below 2^-26 of 2^(-e_i - f_j), far under the float32
//                 rounding of a probability.  Two passes over the key blocks
//                 j <= i: the row maximum and sum of exponentials (float64,
//                 online), then probs_ij = exp(s_ij - max) / sum rounded to
//                 float32; zeros above the diagonal.
//
// score_i8 roles: warps 0-7 epilogue (two threads per query block row, TMEM
// lane = row, each thread 24 of the 48 columns), warp 8 TMA producer (the Q
// digits once, the K digits of each column tile through a two-stage ring),
// warp 9 MMA issuer (accumulators double-buffered in TMEM so a tile's MMAs run
// while the previous tile's epilogue reads).  Every wait is bounded (about
// 2 s); a wait that runs out writes SFA_ERR_TIMEOUT to the status word and the
// CTA drains its copies and MMAs before it frees its tensor memory.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace sfa {

namespace {

constexpr int kDig = 5;                       // digits per value
constexpr int kLevels = 5;                    // digit-pair levels a + b = 0 .. 4
constexpr int kRows = 128;                    // query blocks per CTA (MMA M)
constexpr int kCols = 48;                     // key blocks per column tile (MMA N)
constexpr int kHD = 128;                      // head dim: bytes of one digit row
constexpr uint32_t kQDig = kRows * kHD;       // 16 KB: one Q digit tile
constexpr uint32_t kKDig = kCols * kHD;       // 6 KB: one K digit tile
constexpr uint32_t kKStage = kDig * kKDig;    // 30 KB: a column tile's K digits
constexpr uint32_t kAccCols = kLevels * kCols;  // TMEM columns of one accumulator set
constexpr uint32_t kTmemCols = 512;
constexpr int kThreads = 320;
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr uint64_t kTimeoutNs = 2000000000ull;

enum { B_Q = 0, B_KF = 1, B_KE = 3, B_AF = 5, B_AE = 7, B_DRAIN = 9, NBAR = 10 };  // KF..AE: two each
constexpr uint32_t OFF_K = kDig * kQDig;                  // 80 KB
constexpr uint32_t OFF_BAR = OFF_K + 2 * kKStage;         // 140 KB
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;         // tmem slot, abort flag
constexpr uint32_t OFF_XCHG = OFF_MISC + 16;              // [half][row] (max, sum, flag) for the row merge
constexpr uint32_t SMEM_BYTES = OFF_XCHG + 2 * kRows * 24 + 1024;

// Bounded wait on an mbarrier phase; false if the CTA aborted or the wait ran out.
__device__ bool wait_bar(volatile int* abort_flag, int* status, uint32_t bar, uint32_t parity) {
  if (tc::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (tc::mbar_try_wait(bar, parity)) return true;
    if ((it & 127u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > kTimeoutNs) {
        *abort_flag = 1;
        report(status, SFA_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

__device__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!tc::mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kTimeoutNs) return;
  }
}

// One warp per row of qt (first B * Hq * nb rows) or kbar (then B * Hkv * nb rows).
__global__ void __launch_bounds__(256) score_slices_kernel(ScoreSliceParams p) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const long long nq = (long long)p.B * p.Hq * p.nb, nk = (long long)p.B * p.Hkv * p.nb;
  if (row >= nq + nk) return;
  const bool is_q = row < nq;
  const long long r = is_q ? row : row - nq;
  const double* src = (is_q ? p.qbar : p.kbar) + r * kHD + lane * 4;
  double x[4];
  {
    const double2 u = reinterpret_cast<const double2*>(src)[0];
    const double2 v = reinterpret_cast<const double2*>(src)[1];
    x[0] = u.x; x[1] = u.y; x[2] = v.x; x[3] = v.y;
  }
  if (is_q) {
    const int bh = (int)(r / p.nb);  // b * Hq + h
    const double inv_h = 1.0 / (p.tau[(size_t)bh * 2 + 0] * sqrt((double)kHD));
    const double inv_l = 1.0 / (p.tau[(size_t)bh * 2 + 1] * sqrt((double)kHD));
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] *= ((lane * 4 + e) % (kHD / 2)) < p.band_pairs ? inv_h : inv_l;
  }
  double mx = fmax(fmax(fabs(x[0]), fabs(x[1])), fmax(fabs(x[2]), fabs(x[3])));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  int ex = 0;  // x 2^ex in (-1/2, 1/2)
  if (mx > 0.0) {
    int E;
    frexp(mx, &E);  // mx = f 2^E, f in [1/2, 1)
    ex = -E - 1;
  }
  uint32_t w[kDig] = {0, 0, 0, 0, 0};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    double y = ldexp(x[e], ex);
#pragma unroll
    for (int a = 0; a < kDig; ++a) {
      const double t = y * 128.0;  // exact
      const double d = rint(t);    // |d| <= 64
      y = t - d;                   // exact, |y| <= 1/2
      w[a] |= ((uint32_t)(int)d & 0xFFu) << (8 * e);
    }
  }
  const int bh = (int)(r / p.nb), i = (int)(r % p.nb);
  int8_t* dst = is_q ? p.qd : p.kd;
#pragma unroll
  for (int a = 0; a < kDig; ++a)
    reinterpret_cast<uint32_t*>(dst + (((size_t)bh * kDig + a) * p.nb + i) * kHD)[lane] = w[a];
  if (lane == 0) (is_q ? p.qe : p.ke)[r] = ex;
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
    score_i8_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    ScoreSliceParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  unsigned char* sm = smem_raw + pad;
  const uint32_t sbase = raw + pad;
  const uint32_t bars = sbase + OFF_BAR;
  auto bar = [&](int k) { return bars + 8u * k; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Tile: every head's heaviest (last) row tile first, then the next heaviest, ...
  const int ntr = (p.nb + kRows - 1) / kRows;
  const int nbh = p.B * p.Hq;
  const int rt = ntr - 1 - (int)(blockIdx.x / nbh);
  const int bh = (int)(blockIdx.x % nbh);  // b * Hq + h
  const int b = bh / p.Hq, h = bh % p.Hq, g = h / (p.Hq / p.Hkv);
  const int i0 = rt * kRows;
  const int jend = min(p.nb, i0 + kRows);     // columns [0, jend) hold the tile's causal entries
  const int nct = (jend + kCols - 1) / kCols;  // column tiles per pass

  if (threadIdx.x < 2 * kRows) reinterpret_cast<volatile int*>(sm + OFF_XCHG + 2 * kRows * 16)[threadIdx.x] = 0;
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int k = 0; k < NBAR; ++k) tc::mbar_init(bar(k), (k == B_AE || k == B_AE + 1) ? 256 : 1);
    tc::fence_mbar_init();
  } else if (warp == kProducerWarp && lane == 0) {
    tc::prefetch_tmap(&tmQ);
    tc::prefetch_tmap(&tmK);
  } else if (warp == kMmaWarp) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nu = 2 * nct;  // column tiles over both passes

  if (warp == kProducerWarp) {
    if (lane == 0) {
      int issued = 0;
      bool ok = true;
      tc::mbar_arrive_expect_tx(bar(B_Q), kDig * kQDig);
      for (int a = 0; a < kDig; ++a) tc::tma_load_3d(sbase + a * kQDig, &tmQ, bar(B_Q), 0, i0, bh * kDig + a);
      for (int u = 0; u < nu && ok; ++u) {
        const int s = u & 1;
        if (u >= 2 && !wait_bar(abort_flag, p.status, bar(B_KE + s), ((u >> 1) - 1) & 1)) { ok = false; break; }
        const int ct = u % nct;
        const uint32_t dst = sbase + OFF_K + s * kKStage;
        tc::mbar_arrive_expect_tx(bar(B_KF + s), kKStage);
        for (int a = 0; a < kDig; ++a)
          tc::tma_load_3d(dst + a * kKDig, &tmK, bar(B_KF + s), 0, ct * kCols, (b * p.Hkv + g) * kDig + a);
        ++issued;
      }
      if (*abort_flag) {
        drain_wait(bar(B_Q), 0);
        for (int u = (issued > 2 ? issued - 2 : 0); u < issued; ++u) drain_wait(bar(B_KF + (u & 1)), (u >> 1) & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_s8_s32(kRows, kCols);
      bool ok = wait_bar(abort_flag, p.status, bar(B_Q), 0);
      for (int u = 0; u < nu && ok; ++u) {
        const int s = u & 1, buf = u & 1;
        if (!wait_bar(abort_flag, p.status, bar(B_KF + s), (u >> 1) & 1)) break;
        if (u >= 2 && !wait_bar(abort_flag, p.status, bar(B_AE + buf), ((u >> 1) - 1) & 1)) break;
        tc::tc_fence_after();
        const uint32_t sK = sbase + OFF_K + s * kKStage;
#pragma unroll
        for (int lv = 0; lv < kLevels; ++lv) {
          const uint32_t d = tmem + buf * kAccCols + lv * kCols;
#pragma unroll
          for (int a = 0; a <= lv; ++a) {
            const int bd = lv - a;
#pragma unroll
            for (int kk = 0; kk < kHD / 32; ++kk)
              tc::mma_s8_ss(d, tc::sw128_desc(sbase + a * kQDig + kk * 32, 16, 1024),
                            tc::sw128_desc(sK + bd * kKDig + kk * 32, 16, 1024), idesc, (a > 0 || kk > 0) ? 1u : 0u);
          }
        }
        tc::mma_commit(bar(B_KE + s));
        tc::mma_commit(bar(B_AF + buf));
      }
      tc::mma_commit(bar(B_DRAIN));
      drain_wait(bar(B_DRAIN), 0);
    }
  } else {
    // ------------------------------ epilogue ------------------------------
    const int hf = warp >> 2;                  // columns [24 hf, 24 hf + 24) of a tile
    const int rr = ((warp & 3) << 5) | lane;   // row of the tile = TMEM lane
    const int i = i0 + rr;                     // query block
    const bool live = i < p.nb;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const double rs = ldexp(1.0, -(live ? p.qe[(size_t)bh * p.nb + i] : 0) - 14);
    const int* ke = p.ke + (size_t)(b * p.Hkv + g) * p.nb;
    float* prow = p.probs + ((size_t)bh * p.nb + (live ? i : 0)) * p.nb;
    double m = -INFINITY, l = 0.0, inv = 0.0;
    bool ok = true;
    for (int u = 0; u < nu; ++u) {
      const int buf = u & 1, pass = u / nct, ct = u % nct;
      ok = __all_sync(0xffffffffu, wait_bar(abort_flag, p.status, bar(B_AF + buf), (u >> 1) & 1));
      if (!ok) break;
      tc::tc_fence_after();
      const int j0 = ct * kCols + 24 * hf;
      double sv[24];
#pragma unroll
      for (int c8 = 0; c8 < 3; ++c8) {
        uint32_t v[kLevels][8];
#pragma unroll
        for (int lv = 0; lv < kLevels; ++lv)
          tc::tmem_ld8(tmem + lane_base + buf * kAccCols + lv * kCols + 24 * hf + 8 * c8, v[lv]);
        tc::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int j = j0 + 8 * c8 + e;
          double acc = (double)(int)v[4][e];
          acc = fma(acc, 0x1p-7, (double)(int)v[3][e]);
          acc = fma(acc, 0x1p-7, (double)(int)v[2][e]);
          acc = fma(acc, 0x1p-7, (double)(int)v[1][e]);
          acc = fma(acc, 0x1p-7, (double)(int)v[0][e]);
          const bool in = live && j <= i;  // j <= i < nb
          sv[8 * c8 + e] = in ? acc * rs * ldexp(1.0, -__ldg(ke + min(j, p.nb - 1))) : -INFINITY;
        }
      }
      tc::tc_fence_before();
      tc::mbar_arrive(bar(B_AE + buf));  // the accumulators are in registers: free the buffer
      if (pass == 0) {
        double tm = m;
#pragma unroll
        for (int e = 0; e < 24; ++e) tm = fmax(tm, sv[e]);
        if (tm > -INFINITY) {
          double add = 0.0;
#pragma unroll
          for (int e = 0; e < 24; ++e) add += exp(sv[e] - tm);
          l = (m > -INFINITY ? l * exp(m - tm) : 0.0) + add;
          m = tm;
        }
        if (ct == nct - 1) {
          // Merge the two halves of the row: publish (max, sum), then read the partner's.
          volatile double* xr = reinterpret_cast<volatile double*>(sm + OFF_XCHG);
          volatile int* xf = reinterpret_cast<volatile int*>(sm + OFF_XCHG + 2 * kRows * 16);
          xr[(hf * kRows + rr) * 2 + 0] = m;
          xr[(hf * kRows + rr) * 2 + 1] = l;
          __threadfence_block();
          xf[hf * kRows + rr] = 1;
          const uint64_t t0 = globaltimer_ns();
          for (uint32_t spin = 0; xf[(1 - hf) * kRows + rr] == 0; ++spin) {
            if ((spin & 63u) == 0 && (*abort_flag || globaltimer_ns() - t0 > kTimeoutNs)) {
              if (!*abort_flag) {
                *abort_flag = 1;
                report(p.status, SFA_ERR_TIMEOUT);
              }
              ok = false;
              break;
            }
          }
          if (!__all_sync(0xffffffffu, ok)) break;
          __threadfence_block();
          const double m2 = xr[((1 - hf) * kRows + rr) * 2 + 0], l2 = xr[((1 - hf) * kRows + rr) * 2 + 1];
          const double M = fmax(m, m2);
          const double L = (m > -INFINITY ? l * exp(m - M) : 0.0) + (m2 > -INFINITY ? l2 * exp(m2 - M) : 0.0);
          m = M;
          inv = L > 0.0 ? 1.0 / L : 0.0;
        }
      } else if (live) {
        // Probabilities of this thread's 24 columns; 0 above the diagonal, nothing past nb.
#pragma unroll
        for (int e = 0; e < 24; ++e) {
          const int j = j0 + e;
          if (j < p.nb) prow[j] = (float)(sv[e] > -INFINITY ? exp(sv[e] - m) * inv : 0.0);
        }
      }
    }
    if (!ok && live && hf == 0) {
      // A wait gave up (the call has no status word): the row's probabilities are poisoned.
      for (int j = 0; j < p.nb; ++j) prow[j] = NAN;
    }
    // Columns past the last column tile are above every row's diagonal: zeros, one warp per row.
    const int jz = nct * kCols;
    if (ok && jz < p.nb) {
      for (int r = warp; r < kRows && i0 + r < p.nb; r += 8) {
        float* zr = p.probs + ((size_t)bh * p.nb + i0 + r) * p.nb;
        for (int j = jz + lane; j < p.nb; j += 32) zr[j] = 0.f;
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

cudaError_t launch_score_slices(const ScoreSliceParams& p, cudaStream_t st) {
  const long long rows = (long long)p.B * (p.Hq + p.Hkv) * p.nb;
  score_slices_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_score_i8(const ScoreSliceParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                            cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(score_i8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)(p.B * p.Hq * ((p.nb + kRows - 1) / kRows));
  score_i8_kernel<<<grid, kThreads, SMEM_BYTES, st>>>(tmQ, tmK, p);
  return cudaGetLastError();
}

}  // namespace sfa
