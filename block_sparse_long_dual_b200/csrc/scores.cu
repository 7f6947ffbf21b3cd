// Block-importance estimate of "Prism: Spectral-Aware Block-Sparse Attention"
// (§2 mean pooling under RoPE, §3.1 dual-band pooling, §3.2 energy temperature,
// §5 block-level matrix products only).
//
// Three kernels, launched in order on one stream:
//   rope_pool_energy  HBM stream over Q and K: RoPE, rotated copy, per-block
//                     mean vectors and per-band energies (one CTA per block
//                     and group of heads, each head's block staged by bulk
//                     asynchronous copies).
//   band_temperature  per (batch, Q head): reduce the energies to tau^H, tau^L.
//   block_score_softmax  calibrated block logits (float64 tensor-core MMAs)
//                     and the causal row softmax, both in float64; in the
//                     FUSED instantiation each row's selection follows in the
//                     same warp (select_row.cuh), so the probabilities need
//                     not reach device memory.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "select_row.cuh"

namespace sfa {

// ---------------------------------------------------------------------------
// rope_pool_energy
// One CTA per (batch, block, group of heads).  The cos/sin slice of the block
// (shared by every head) is read once into registers; the block's rows of Q or
// K of each head (contiguous, 32 KB for bf16 d = 128) stream through an
// NS-stage shared-memory ring filled by bulk asynchronous copies (mbarrier per
// stage), so HBM reads stay in flight without holding registers.  Per head:
// CH = D/16 threads cover one token (each owns 8 rotary pairs), 256 / CH
// tokens per pass; RoPE in float32, the rotated row written back (input dtype,
// round to nearest even), per-thread partial sums reduced across threads in
// float64 to the block mean and the per-band energies.
// ---------------------------------------------------------------------------
template <typename T, int D, int PASSES, int NS>
__global__ void __launch_bounds__(256, (sizeof(T) == 2 ? 2 : 1)) rope_pool_energy_kernel(RopePoolParams p, int heads_per_cta) {
  constexpr int CH = D / 16;
  constexpr int TPP = 256 / CH;  // tokens per pass
  constexpr int NW = 8;
  constexpr int BLK = TPP * PASSES;
  constexpr uint32_t XBYTES = BLK * D * sizeof(T);
  __shared__ double red[NW][D];
  __shared__ double ered[NW][4];
  __shared__ __align__(8) uint64_t bars[NS];
  extern __shared__ __align__(128) unsigned char smem_dyn[];  // [NS][BLK][D] elements

  const int heads = p.Hq + p.Hkv;
  const int ngroups = (heads + heads_per_cta - 1) / heads_per_cta;
  int bid = blockIdx.x;
  const int hg = bid % ngroups;
  bid /= ngroups;
  const int j = bid % p.nb;
  const int b = bid / p.nb;
  const int h0 = hg * heads_per_cta;
  const int h1 = min(heads, h0 + heads_per_cta);
  const int nh = h1 - h0;

  const int tid = threadIdx.x;
  const int c = tid % CH;
  const int tk = tid / CH;
  const int lane = tid & 31, warp = tid >> 5;

  auto src_of = [&](int head) -> const T* {
    const bool is_q = head < p.Hq;
    const int hh = is_q ? head : head - p.Hq;
    const int H = is_q ? p.Hq : p.Hkv;
    const size_t row0 = ((size_t)(b * H + hh) * p.L) + (size_t)j * BLK;
    return static_cast<const T*>(is_q ? p.Q : p.K) + row0 * D;
  };
  auto stage_ptr = [&](int st) { return reinterpret_cast<T*>(smem_dyn + (size_t)st * XBYTES); };

  if (tid == 0) {
    for (int st = 0; st < NS; ++st)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"((uint32_t)__cvta_generic_to_shared(&bars[st]))
                   : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int st = 0; st < NS && st < nh; ++st)
      arm_and_load((uint32_t)__cvta_generic_to_shared(&bars[st]),
                   (uint32_t)__cvta_generic_to_shared(stage_ptr(st)), src_of(h0 + st), XBYTES);
  }

  // The block's cos/sin slice, once per CTA: pairs [8c, 8c+8) of tokens ps*TPP + tk.
  float csv[PASSES][8], snv[PASSES][8];
#pragma unroll
  for (int ps = 0; ps < PASSES; ++ps) {
    const size_t pos = (size_t)j * BLK + ps * TPP + tk;
    if (p.apply) {
      load8(p.cos + pos * (D / 2) + c * 8, csv[ps]);
      load8(p.sin + pos * (D / 2) + c * 8, snv[ps]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) { csv[ps][e] = 1.f; snv[ps][e] = 0.f; }
    }
  }
  __syncthreads();  // barriers initialised

  for (int q = 0; q < nh; ++q) {
    const int head = h0 + q;
    const int st = q % NS;
    const bool landed = wait_parity_bounded((uint32_t)__cvta_generic_to_shared(&bars[st]), (q / NS) & 1);
    const bool is_q = head < p.Hq;
    const int hh = is_q ? head : head - p.Hq;
    const int H = is_q ? p.Hq : p.Hkv;
    const size_t row0 = ((size_t)(b * H + hh) * p.L) + (size_t)j * BLK;
    void* xdst = p.write_rot ? (is_q ? p.Qr : p.Kr) : nullptr;  // Qr may be NULL: Q rotated on load later
    T* xr = xdst != nullptr ? static_cast<T*>(xdst) + row0 * D : nullptr;
    const T* xs = stage_ptr(st);

    float slo[8], shi[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) slo[e] = shi[e] = 0.f;
    double eh = 0.0, el = 0.0;
#pragma unroll
    for (int ps = 0; ps < PASSES; ++ps) {
      const int t = ps * TPP + tk;
      float lo[8], hi[8];
      load8_smem(xs + (size_t)t * D + c * 8, lo);
      load8_smem(xs + (size_t)t * D + D / 2 + c * 8, hi);
      if (p.apply) {
#pragma unroll
        for (int e = 0; e < 8; ++e) rope_pair(lo[e], hi[e], csv[ps][e], snv[ps][e], lo[e], hi[e]);
        if (xr != nullptr) {
          store8(xr + (size_t)t * D + c * 8, lo);
          store8(xr + (size_t)t * D + D / 2 + c * 8, hi);
        }
      }
      float ph = 0.f, pl = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        slo[e] += lo[e];
        shi[e] += hi[e];
        const float en = fmaf(lo[e], lo[e], hi[e] * hi[e]);
        if (c * 8 + e < p.band_pairs) ph += en; else pl += en;
      }
      eh += ph;
      el += pl;
    }

    // Cross-thread reduction in float64: lanes with equal c hold the same dims.
    double dlo[8], dhi[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) { dlo[e] = slo[e]; dhi[e] = shi[e]; }
#pragma unroll
    for (int off = CH; off < 32; off <<= 1) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        dlo[e] += __shfl_xor_sync(0xffffffffu, dlo[e], off);
        dhi[e] += __shfl_xor_sync(0xffffffffu, dhi[e], off);
      }
    }
    if (lane < CH) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        red[warp][lane * 8 + e] = dlo[e];
        red[warp][D / 2 + lane * 8 + e] = dhi[e];
      }
    }
    double deh = eh, del = el;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      deh += __shfl_xor_sync(0xffffffffu, deh, off);
      del += __shfl_xor_sync(0xffffffffu, del, off);
    }
    if (lane == 0) { ered[warp][0] = deh; ered[warp][1] = del; }
    __syncthreads();  // stage st fully read; partial sums visible
    if (tid == 0 && q + NS < nh)
      arm_and_load((uint32_t)__cvta_generic_to_shared(&bars[st]), (uint32_t)__cvta_generic_to_shared(stage_ptr(st)),
                   src_of(h0 + q + NS), XBYTES);

    // One thread per dim: block mean, pooled energy per band.
    double ph = 0.0, pl = 0.0;
    if (tid < D) {
      double sacc = 0.0;
#pragma unroll
      for (int w = 0; w < NW; ++w) sacc += red[w][tid];
      const double mean = landed ? sacc / (double)BLK : (double)NAN;  // a copy that never landed poisons tau
      double* out = (is_q ? p.qbar + ((size_t)(b * p.Hq + hh) * p.nb + j) * D
                          : p.kbar + ((size_t)(b * p.Hkv + hh) * p.nb + j) * D);
      out[tid] = mean;
      const int m = tid % (D / 2);
      if (m < p.band_pairs) ph = mean * mean; else pl = mean * mean;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      ph += __shfl_xor_sync(0xffffffffu, ph, off);
      pl += __shfl_xor_sync(0xffffffffu, pl, off);
    }
    if (lane == 0) { ered[warp][2] = ph; ered[warp][3] = pl; }
    __syncthreads();
    if (tid < 4) {
      double sacc = 0.0;
#pragma unroll
      for (int w = 0; w < NW; ++w) sacc += ered[w][tid];
      p.energy[((size_t)(b * heads + head) * p.nb + j) * 4 + tid] = landed ? sacc : (double)NAN;
    }
    __syncthreads();  // red / ered free for the next head
  }
}

// ---------------------------------------------------------------------------
// band_temperature: tau^b = max(rho^b(Q_h) * rho^b(K_g), 1e-6),
// rho = sqrt(mean_j ||xbar_j^b||^2 / mean_t ||x_t^b||^2), 1 for a band without energy;
// with SFA_RELATIVE_CALIB tau^H / tau^L and 1.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) band_temperature_kernel(TauParams p) {
  const int h = blockIdx.x % p.Hq;
  const int b = blockIdx.x / p.Hq;
  const int g = h / (p.Hq / p.Hkv);
  const int heads = p.Hq + p.Hkv;
  const double* eq = p.energy + (size_t)(b * heads + h) * p.nb * 4;
  const double* ek = p.energy + (size_t)(b * heads + p.Hq + g) * p.nb * 4;
  double acc[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) acc[q] = 0.0;
  for (int j = threadIdx.x; j < p.nb; j += blockDim.x) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      acc[q] += eq[(size_t)j * 4 + q];
      acc[4 + q] += ek[(size_t)j * 4 + q];
    }
  }
  __shared__ double red[8][8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc[q] += __shfl_xor_sync(0xffffffffu, acc[q], off);
    if (lane == 0) red[warp][q] = acc[q];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double tau[2] = {1.0, 1.0};  // band H, band L
    if (!(p.flags & SFA_NO_CALIB)) {
      for (int band = 0; band < 2; ++band) {
        double tq = 0, pq = 0, tk = 0, pk = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
          tq += red[w][band]; pq += red[w][2 + band];
          tk += red[w][4 + band]; pk += red[w][6 + band];
        }
        const double etq = tq / (double)p.L, epq = pq / (double)p.nb;
        const double etk = tk / (double)p.L, epk = pk / (double)p.nb;
        const double rq = etq > 0.0 ? sqrt(epq / etq) : 1.0;
        const double rk = etk > 0.0 ? sqrt(epk / etk) : 1.0;
        tau[band] = fmax(rq * rk, 1e-6);
      }
      if (p.flags & SFA_RELATIVE_CALIB) {
        // Alternative reading: only the high band's amplitude relative to the low band is restored.
        tau[0] = (p.flags & SFA_SINGLE_BAND) ? 1.0 : tau[0] / tau[1];
        tau[1] = 1.0;
      }
    }
    p.tau[(size_t)(b * p.Hq + h) * 2 + 0] = tau[0];
    p.tau[(size_t)(b * p.Hq + h) * 2 + 1] = tau[1];
  }
}

// ---------------------------------------------------------------------------
// block_score_softmax
// CTA = RT query-block rows of one (b, h).  The calibrated logits of the rows
// are kept as a float64 strip [RT][nb] in shared memory, computed on the
// float64 tensor cores (mma.sync m8n8k4 .f64: tcgen05 has no float64 kind):
// column steps of 256 key blocks, each warp owns 4 column tiles of 8 and all
// RT/8 row tiles, the head dim in k-steps of 4.  A fragments (calibrated query
// means) come from shared memory, B fragments (key means) straight from L2,
// prefetched one k-step ahead.  Column tiles past the causal diagonal are
// skipped.  Then the causal row softmax in float64, one warp per row.
// Everything is float64 because the calibration 1/tau amplifies the pooled
// logits: float32 sums of logits of magnitude ~20 already err by ~1e-6.
//
// Alternative readings (flags):
//   SFA_BLOCK_TAU  per-block temperature: the query means of row i are scaled
//                  by 1/rho^b_i(Q) and each key mean element by 1/rho^b_j(K)
//                  as its fragment is loaded (rho from the block energies).
//   SFA_BAND_MAX   one GEMM pass per band (the other band's query dims zeroed),
//                  each with its own causal softmax; band H's probabilities
//                  wait in a float32 strip [RT][nb] until band L's pass takes
//                  the elementwise maximum and renormalises.
// ---------------------------------------------------------------------------
// Retained amplitude of one block and band: sqrt(||xbar||^2 / mean_t ||x_t||^2),
// floored at 1e-3, 1 when the block's band has no energy.
__device__ __forceinline__ double block_rho(double tok, double pool, int block) {
  return tok == 0.0 ? 1.0 : fmax(sqrt(pool * (double)block / tok), 1e-3);
}

__device__ __forceinline__ void dmma_8x8x4(double (&c)[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(c[0]), "+d"(c[1])
               : "d"(a), "d"(b));
}

template <int RT, int D, int NPL, bool FUSED>
__global__ void __launch_bounds__(256, 1) block_score_softmax_kernel(ScoreParams p) {
  constexpr int RTL = RT / 8;             // row tiles
  constexpr int CS = 256;                 // columns per step
  constexpr int CTW = 4;                  // column tiles per warp (8 warps x 4 x 8 = 256)
  constexpr int QLD = D + 4;              // padded row of the query tile (doubles)
  constexpr int KS = D / 4;               // k-steps
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double* strip = reinterpret_cast<double*>(smem_raw);                 // [RT][nb]
  double* qs = strip + (size_t)RT * p.nb;                               // [RT][QLD]
  float* pstrip = reinterpret_cast<float*>(qs + RT * QLD);              // [RT][nb], band-max only

  const int ntiles = (p.nb + RT - 1) / RT;
  const int tile = ntiles - 1 - (int)blockIdx.x;  // heaviest rows first
  const int h = blockIdx.y, b = blockIdx.z;
  const int g = h / (p.Hq / p.Hkv);
  const int i0 = tile * RT;
  const int rows = min(RT, p.nb - i0);
  const int jend = i0 + rows;  // columns [0, jend)
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;  // mma fragment coordinates

  const bool block_tau = (p.flags & SFA_BLOCK_TAU) != 0;
  const bool two = (p.flags & SFA_BAND_MAX) && p.band_pairs > 0 && p.band_pairs < D / 2;
  const int heads = p.Hq + p.Hkv;
  const double* tau = p.tau + (size_t)(b * p.Hq + h) * 2;
  const double inv_h = 1.0 / (tau[0] * sqrt((double)D));
  const double inv_l = 1.0 / (tau[1] * sqrt((double)D));
  const double* qsrc = p.qbar + ((size_t)(b * p.Hq + h) * p.nb + i0) * D;
  const double* ksrc = p.kbar + (size_t)(b * p.Hkv + g) * p.nb * D;
  const double* eq = p.energy + ((size_t)(b * heads + h) * p.nb) * 4;
  const double* ek = p.energy + ((size_t)(b * heads + p.Hq + g) * p.nb) * 4;

  for (int pass = 0; pass < (two ? 2 : 1); ++pass) {
    // Calibrated, pre-scaled query block means: q~ = qbar / (tau^band * sqrt(d)) (per-block
    // rho^band_i(Q) instead of tau with SFA_BLOCK_TAU); with SFA_BAND_MAX pass 0 keeps band H's
    // dims only and pass 1 band L's.
    for (int e = tid; e < D * RT; e += 256) {
      const int r = e / D, d = e % D;
      const bool hb = (d % (D / 2)) < p.band_pairs;
      double sc;
      if (block_tau) {
        const double* er = eq + (size_t)min(i0 + r, p.nb - 1) * 4;
        sc = 1.0 / (block_rho(er[hb ? 0 : 1], er[hb ? 2 : 3], p.block) * sqrt((double)D));
      } else {
        sc = hb ? inv_h : inv_l;
      }
      if (two && hb != (pass == 0)) sc = 0.0;
      qs[r * QLD + d] = (r < rows) ? qsrc[(size_t)r * D + d] * sc : 0.0;
    }
    __syncthreads();

    for (int col0 = 0; col0 < jend; col0 += CS) {
      // this warp's column tiles: col0 + (warp * CTW + ct) * 8 .. + 8
      int ntl = 0;
#pragma unroll
      for (int ct = 0; ct < CTW; ++ct) ntl += (col0 + (warp * CTW + ct) * 8 < jend) ? 1 : 0;
      if (ntl > 0) {
        double acc[RTL][CTW][2];
#pragma unroll
        for (int rt = 0; rt < RTL; ++rt)
#pragma unroll
          for (int ct = 0; ct < CTW; ++ct) acc[rt][ct][0] = acc[rt][ct][1] = 0.0;
        // B fragment of column tile ct at k-step ks: kbar[col][4 ks + tq], col = tile start + gq.
        const double* kptr[CTW];
        double kih[CTW], kil[CTW];  // 1 / rho^band_col(K) with SFA_BLOCK_TAU, else 1
#pragma unroll
        for (int ct = 0; ct < CTW; ++ct) {
          const int col = min(col0 + (warp * CTW + ct) * 8 + gq, p.nb - 1);
          kptr[ct] = ksrc + (size_t)col * D + tq;
          kih[ct] = kil[ct] = 1.0;
          if (block_tau) {
            const double* er = ek + (size_t)col * 4;
            kih[ct] = 1.0 / block_rho(er[0], er[2], p.block);
            kil[ct] = 1.0 / block_rho(er[1], er[3], p.block);
          }
        }
        // B fragments in batches of KB k-steps, double-buffered in registers: the next batch's L2
        // loads are in flight while this batch's MMAs run.
        constexpr int KB = 4;
        constexpr int NKB = KS / KB;
        double bb[2][KB][CTW];
        auto load_batch = [&](int kb, double (&dst)[KB][CTW]) {
#pragma unroll
          for (int u = 0; u < KB; ++u) {
            const int ks = kb * KB + u;
            const bool hb = ((4 * ks + tq) % (D / 2)) < p.band_pairs;
#pragma unroll
            for (int ct = 0; ct < CTW; ++ct) dst[u][ct] = __ldg(kptr[ct] + 4 * ks) * (hb ? kih[ct] : kil[ct]);
          }
        };
        load_batch(0, bb[0]);
#pragma unroll
        for (int kb = 0; kb < NKB; ++kb) {
          if (kb + 1 < NKB) load_batch(kb + 1, bb[(kb + 1) & 1]);
#pragma unroll
          for (int u = 0; u < KB; ++u) {
            const int ks = kb * KB + u;
            double a[RTL];
#pragma unroll
            for (int rt = 0; rt < RTL; ++rt) a[rt] = qs[(rt * 8 + gq) * QLD + 4 * ks + tq];
#pragma unroll
            for (int ct = 0; ct < CTW; ++ct) {
              if (ct < ntl) {
#pragma unroll
                for (int rt = 0; rt < RTL; ++rt) dmma_8x8x4(acc[rt][ct], a[rt], bb[kb & 1][u][ct]);
              }
            }
          }
        }
        // C fragment: (row gq, cols 2 tq, 2 tq + 1) of each tile
#pragma unroll
        for (int rt = 0; rt < RTL; ++rt) {
          const int rr = rt * 8 + gq;
#pragma unroll
          for (int ct = 0; ct < CTW; ++ct) {
            const int col = col0 + (warp * CTW + ct) * 8 + 2 * tq;
            if (ct < ntl) {  // scalar stores: nb may be odd, so a row need not start 16-byte aligned
              if (col < jend) strip[(size_t)rr * p.nb + col] = acc[rt][ct][0];
              if (col + 1 < jend) strip[(size_t)rr * p.nb + col + 1] = acc[rt][ct][1];
            }
          }
        }
      }
    }
    __syncthreads();
    if (two && pass == 0) {
      // Band H's causal softmax, kept as float32 probabilities for pass 1.
      for (int r = warp; r < rows; r += 8) {
        const int i = i0 + r;
        const double* srow = strip + (size_t)r * p.nb;
        double m = -INFINITY;
        for (int jj = lane; jj <= i; jj += 32) m = fmax(m, srow[jj]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, off));
        double sum = 0.0;
        for (int jj = lane; jj <= i; jj += 32) sum += exp(srow[jj] - m);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        const double inv = 1.0 / sum;
        float* prow = pstrip + (size_t)r * p.nb;
        for (int jj = lane; jj <= i; jj += 32) prow[jj] = (float)(exp(srow[jj] - m) * inv);
      }
      __syncthreads();  // strip free for band L; pstrip complete
    }
  }

  // Causal row softmax in float64, one warp per row.
  for (int r = warp; r < rows; r += 8) {
    const int i = i0 + r;
    double* srow = strip + (size_t)r * p.nb;
    double m = -INFINITY;
    for (int jj = lane; jj <= i; jj += 32) m = fmax(m, srow[jj]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, off));
    double sum = 0.0;
    for (int jj = lane; jj <= i; jj += 32) {
      const double e = exp(srow[jj] - m);
      srow[jj] = e;
      sum += e;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    double inv = 1.0 / sum;
    if (two) {
      // Band max: c_j = max(p^H_j, p^L_j), renormalised over j <= i.
      const float* prow = pstrip + (size_t)r * p.nb;
      double z = 0.0;
      for (int jj = lane; jj <= i; jj += 32) {
        const double c = fmax((double)prow[jj], srow[jj] * inv);
        srow[jj] = c;
        z += c;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
      inv = 1.0 / z;
    }
    const size_t rowid = (size_t)(b * p.Hq + h) * p.nb + i;
    if (p.probs != nullptr) {
      float* prow = p.probs + rowid * p.nb;
      for (int jj = lane; jj < p.nb; jj += 32) prow[jj] = (jj <= i) ? (float)(srow[jj] * inv) : 0.f;
    }
    if constexpr (FUSED) {
      // Select on exactly the float32 probabilities the unfused path would write.
      __syncwarp();
      const int n = select_row_warp<NPL>([&](int j) { return (float)(srow[j] * inv); }, i, p.k, p.mass, p.flags,
                                         p.idx + rowid * p.kmax, p.kmax);
      if (lane == 0) p.counts[rowid] = n;
    }
  }
}

// ---------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------
template <typename T, int D, int PASSES>
static cudaError_t launch_rope_pool_tdp(const RopePoolParams& p, cudaStream_t st) {
  constexpr int NS = sizeof(T) == 2 ? 3 : 2;  // ring stages of one head's block rows
  const size_t smem = (size_t)NS * (256 / (D / 16)) * PASSES * D * sizeof(T);
  auto kern = rope_pool_energy_kernel<T, D, PASSES, NS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  // Enough CTAs for about four waves of two CTAs on each of 148 SMs (bf16: two CTAs of a two-stage
  // ring share an SM); each CTA reads the table slice once for its heads.
  const int heads = p.Hq + p.Hkv;
  const long long blocks = (long long)p.B * p.nb;
  int groups = (int)((8LL * 148 + blocks - 1) / blocks);
  groups = groups < 1 ? 1 : (groups > heads ? heads : groups);
  const int per = (heads + groups - 1) / groups;
  groups = (heads + per - 1) / per;
  const unsigned grid = (unsigned)(blocks * groups);
  kern<<<grid, 256, smem, st>>>(p, per);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_rope_pool_t(const RopePoolParams& p, int D, cudaStream_t st) {
  // tokens per pass: 256 / (D / 16) = 32 (D = 128) or 64 (D = 64)
  if (D == 128) return p.block == 128 ? launch_rope_pool_tdp<T, 128, 4>(p, st) : launch_rope_pool_tdp<T, 128, 2>(p, st);
  return p.block == 128 ? launch_rope_pool_tdp<T, 64, 2>(p, st) : launch_rope_pool_tdp<T, 64, 1>(p, st);
}

cudaError_t launch_rope_pool_energy(const RopePoolParams& p, int dtype, int D, cudaStream_t st) {
  if (dtype == SFA_BF16) return launch_rope_pool_t<__nv_bfloat16>(p, D, st);
  return launch_rope_pool_t<float>(p, D, st);
}

cudaError_t launch_band_temperature(const TauParams& p, cudaStream_t st) {
  band_temperature_kernel<<<p.B * p.Hq, 256, 0, st>>>(p);
  return cudaGetLastError();
}

int score_rows_per_cta(int nb) { return nb <= 1024 ? 16 : 8; }

size_t score_smem_bytes(int nb, int D, bool band_max) {
  const int RT = score_rows_per_cta(nb);
  return ((size_t)RT * nb + (size_t)RT * (D + 4)) * sizeof(double) + (band_max ? (size_t)RT * nb * sizeof(float) : 0);
}

template <int RT, int D, int NPL, bool FUSED>
static cudaError_t launch_score_t(const ScoreParams& p, cudaStream_t st) {
  const size_t smem =
      score_smem_bytes(p.nb, D, (p.flags & SFA_BAND_MAX) && p.band_pairs > 0 && p.band_pairs < D / 2);
  auto kern = block_score_softmax_kernel<RT, D, NPL, FUSED>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((p.nb + RT - 1) / RT, p.Hq, p.B);
  kern<<<grid, 256, smem, st>>>(p);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_score_d(const ScoreParams& p, cudaStream_t st) {
  if (p.counts == nullptr) {
    return score_rows_per_cta(p.nb) == 16 ? launch_score_t<16, D, 1, false>(p, st)
                                          : launch_score_t<8, D, 1, false>(p, st);
  }
  if (p.nb <= 32) return launch_score_t<16, D, 1, true>(p, st);
  if (p.nb <= 64) return launch_score_t<16, D, 2, true>(p, st);
  if (p.nb <= 128) return launch_score_t<16, D, 4, true>(p, st);
  if (p.nb <= 256) return launch_score_t<16, D, 8, true>(p, st);
  if (p.nb <= 512) return launch_score_t<16, D, 16, true>(p, st);
  if (p.nb <= 1024) return launch_score_t<16, D, 32, true>(p, st);
  return launch_score_t<8, D, 64, true>(p, st);
}

cudaError_t launch_block_score_softmax(const ScoreParams& p, int D, cudaStream_t st) {
  return D == 128 ? launch_score_d<128>(p, st) : launch_score_d<64>(p, st);
}

}  // namespace sfa
