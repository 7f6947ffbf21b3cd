// Block-importance estimate of "Prism: Spectral-Aware Block-Sparse Attention"
// (§2 mean pooling under RoPE, §3.1 dual-band pooling, §3.2 energy temperature,
// §5 block-level matrix products only).
//
// Three kernels, launched in order on one stream:
//   rope_pool_energy  HBM stream over Q and K: RoPE, rotated copy, per-block
//                     mean vectors and per-band energies (one CTA per block
//                     and head).
//   band_temperature  per (batch, Q head): reduce the energies to tau^H, tau^L.
//   block_score_softmax  calibrated block logits and the causal row softmax,
//                     both in float64.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace sfa {

// ---------------------------------------------------------------------------
// rope_pool_energy
// Thread map: CH = D/16 threads cover one token (each owns 8 dims of the low
// half and the matching 8 dims of the high half, i.e. 8 rotary pairs);
// 256 / CH tokens per pass; block / (256 / CH) passes.
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(256) rope_pool_energy_kernel(RopePoolParams p) {
  constexpr int CH = D / 16;
  constexpr int TPP = 256 / CH;  // tokens per pass
  constexpr int NW = 8;
  __shared__ double red[NW][D];
  __shared__ double ered[NW][4];

  const int heads = p.Hq + p.Hkv;
  int bid = blockIdx.x;
  const int head = bid % heads;
  bid /= heads;
  const int j = bid % p.nb;
  const int b = bid / p.nb;
  const bool is_q = head < p.Hq;
  const int hh = is_q ? head : head - p.Hq;
  const int H = is_q ? p.Hq : p.Hkv;
  const size_t row0 = ((size_t)(b * H + hh) * p.L) + (size_t)j * p.block;
  const T* x = static_cast<const T*>(is_q ? p.Q : p.K) + row0 * D;
  T* xr = p.write_rot ? static_cast<T*>(is_q ? p.Qr : p.Kr) + row0 * D : nullptr;

  const int tid = threadIdx.x;
  const int c = tid % CH;
  const int tk = tid / CH;
  const int lane = tid & 31, warp = tid >> 5;

  float slo[8], shi[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) slo[e] = shi[e] = 0.f;
  double eh = 0.0, el = 0.0;

  const int passes = p.block / TPP;
  for (int ps = 0; ps < passes; ++ps) {
    const int t = ps * TPP + tk;          // token within the block
    const size_t pos = (size_t)j * p.block + t;  // absolute position
    float lo[8], hi[8];
    load8(x + (size_t)t * D + c * 8, lo);
    load8(x + (size_t)t * D + D / 2 + c * 8, hi);
    if (p.apply) {
      float cs[8], sn[8];
      load8(p.cos + pos * (D / 2) + c * 8, cs);
      load8(p.sin + pos * (D / 2) + c * 8, sn);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float a = lo[e], bb = hi[e];
        lo[e] = fmaf(a, cs[e], -bb * sn[e]);
        hi[e] = fmaf(bb, cs[e], a * sn[e]);
      }
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
  __syncthreads();

  // One thread per dim: block mean, pooled energy per band.
  double ph = 0.0, pl = 0.0;
  if (tid < D) {
    double s = 0.0;
#pragma unroll
    for (int w = 0; w < NW; ++w) s += red[w][tid];
    const double mean = s / (double)p.block;
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
  __syncthreads();  // everyone has read red / ered partials of the token energy
  if (lane == 0) { ered[warp][2] = ph; ered[warp][3] = pl; }
  __syncthreads();
  if (tid < 4) {
    double s = 0.0;
#pragma unroll
    for (int w = 0; w < NW; ++w) s += ered[w][tid];
    p.energy[((size_t)(b * heads + head) * p.nb + j) * 4 + tid] = s;
  }
}

// ---------------------------------------------------------------------------
// band_temperature: tau^b = max(rho^b(Q_h) * rho^b(K_g), 1e-6),
// rho = sqrt(mean_j ||xbar_j^b||^2 / mean_t ||x_t^b||^2), 1 for an empty band.
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
  if (threadIdx.x < 2) {
    const int band = threadIdx.x;  // 0 = H, 1 = L
    double tq = 0, pq = 0, tk = 0, pk = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
      tq += red[w][band]; pq += red[w][2 + band];
      tk += red[w][4 + band]; pk += red[w][6 + band];
    }
    double tau = 1.0;
    if (!(p.flags & SFA_NO_CALIB)) {
      const double etq = tq / (double)p.L, epq = pq / (double)p.nb;
      const double etk = tk / (double)p.L, epk = pk / (double)p.nb;
      const double rq = etq > 0.0 ? sqrt(epq / etq) : 1.0;
      const double rk = etk > 0.0 ? sqrt(epk / etk) : 1.0;
      tau = fmax(rq * rk, 1e-6);
    }
    p.tau[(size_t)(b * p.Hq + h) * 2 + band] = tau;
  }
}

// ---------------------------------------------------------------------------
// block_score_softmax
// CTA = RT query-block rows of one (b, h).  The calibrated logits of the rows
// are kept as a float64 strip [RT][nb] in shared memory.  Column steps of
// CS = 256 keys; the head dim in chunks of DC staged transposed in shared
// memory (float64), the next chunk prefetched into registers while the current
// one is used.  Thread tile: TR rows x 2 columns of float64 FMAs (the query
// operands are warp-uniform broadcasts).
// Everything is float64 because the calibration 1/tau amplifies the pooled
// logits: float32 sums of logits of magnitude ~20 already err by ~1e-6.
// ---------------------------------------------------------------------------
template <int RT, int D>
__global__ void __launch_bounds__(256) block_score_softmax_kernel(ScoreParams p) {
  constexpr int TC = 2;
  constexpr int CS = 256;                 // columns per step: one per thread when staging
  constexpr int CG = CS / TC;             // column groups
  constexpr int RG = 256 / CG;            // row groups
  constexpr int TR = RT / RG;             // rows per thread
  constexpr int DC = 16;                  // head-dim chunk
  constexpr int NCH = D / DC;
  static_assert(TR * RG == RT && TR % 2 == 0, "tile");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double* strip = reinterpret_cast<double*>(smem_raw);                 // [RT][nb]
  double* qT = strip + (size_t)RT * p.nb;                               // [D][RT]
  double* kT = qT + D * RT;                                             // [DC][CS]

  const int ntiles = (p.nb + RT - 1) / RT;
  const int tile = ntiles - 1 - (int)blockIdx.x;  // heaviest rows first
  const int h = blockIdx.y, b = blockIdx.z;
  const int g = h / (p.Hq / p.Hkv);
  const int i0 = tile * RT;
  const int rows = min(RT, p.nb - i0);
  const int jend = i0 + rows;  // columns [0, jend)
  const int tid = threadIdx.x;
  const int rg = tid / CG, cg = tid % CG;

  // Calibrated, pre-scaled query block means: q~ = qbar / (tau^band * sqrt(d)).
  const double* tau = p.tau + (size_t)(b * p.Hq + h) * 2;
  const double inv_h = 1.0 / (tau[0] * sqrt((double)D));
  const double inv_l = 1.0 / (tau[1] * sqrt((double)D));
  const double* qsrc = p.qbar + ((size_t)(b * p.Hq + h) * p.nb + i0) * D;
  for (int e = tid; e < D * RT; e += 256) {
    const int r = e / D, d = e % D;
    const double s = ((d % (D / 2)) < p.band_pairs) ? inv_h : inv_l;
    qT[d * RT + r] = (r < rows) ? qsrc[(size_t)r * D + d] * s : 0.0;
  }
  const double* ksrc = p.kbar + (size_t)(b * p.Hkv + g) * p.nb * D;

  // Register stage of one K-bar chunk: column col0 + tid, dims [dc, dc + DC).
  double2 stage[DC / 2];
  auto fetch = [&](int col0, int dc) {
    const int col = col0 + tid;
    const double2* src = reinterpret_cast<const double2*>(ksrc + (size_t)col * D + dc);
#pragma unroll
    for (int v = 0; v < DC / 2; ++v) stage[v] = col < jend ? __ldg(src + v) : make_double2(0.0, 0.0);
  };

  fetch(0, 0);
  for (int col0 = 0; col0 < jend; col0 += CS) {
    double acc[TR][TC];
#pragma unroll
    for (int r = 0; r < TR; ++r)
#pragma unroll
      for (int q = 0; q < TC; ++q) acc[r][q] = 0.0;
    for (int ch = 0; ch < NCH; ++ch) {
      __syncthreads();  // previous chunk consumed
#pragma unroll
      for (int v = 0; v < DC / 2; ++v) {
        kT[(v * 2 + 0) * CS + tid] = stage[v].x;
        kT[(v * 2 + 1) * CS + tid] = stage[v].y;
      }
      __syncthreads();
      // prefetch the next chunk (next column step after the last chunk)
      if (ch + 1 < NCH) fetch(col0, (ch + 1) * DC);
      else if (col0 + CS < jend) fetch(col0 + CS, 0);
      const int dc = ch * DC;
#pragma unroll
      for (int dd = 0; dd < DC; ++dd) {
        double qv[TR];
#pragma unroll
        for (int r = 0; r < TR; r += 2) {
          const double2 t = *reinterpret_cast<const double2*>(qT + (dc + dd) * RT + rg * TR + r);
          qv[r] = t.x; qv[r + 1] = t.y;
        }
        const double2 kv = *reinterpret_cast<const double2*>(kT + dd * CS + cg * TC);
#pragma unroll
        for (int r = 0; r < TR; ++r) {
          acc[r][0] = fma(qv[r], kv.x, acc[r][0]);
          acc[r][1] = fma(qv[r], kv.y, acc[r][1]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < TR; ++r) {
      const int rr = rg * TR + r;
#pragma unroll
      for (int q = 0; q < TC; ++q) {
        const int col = col0 + cg * TC + q;
        if (col < jend) strip[(size_t)rr * p.nb + col] = acc[r][q];
      }
    }
  }
  __syncthreads();

  // Causal row softmax in float64, one warp per row.
  const int lane = tid & 31, warp = tid >> 5;
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
    const double inv = 1.0 / sum;
    float* prow = p.probs + ((size_t)(b * p.Hq + h) * p.nb + i) * p.nb;
    for (int jj = lane; jj < p.nb; jj += 32) prow[jj] = (jj <= i) ? (float)(srow[jj] * inv) : 0.f;
  }
}

// ---------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------
template <typename T>
static cudaError_t launch_rope_pool_t(const RopePoolParams& p, int D, cudaStream_t st) {
  const unsigned grid = (unsigned)((size_t)p.B * p.nb * (p.Hq + p.Hkv));
  if (D == 128) rope_pool_energy_kernel<T, 128><<<grid, 256, 0, st>>>(p);
  else rope_pool_energy_kernel<T, 64><<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
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

size_t score_smem_bytes(int nb, int D) {
  const int RT = score_rows_per_cta(nb);
  return ((size_t)RT * nb + (size_t)D * RT + (size_t)16 * 256) * sizeof(double);
}

template <int RT, int D>
static cudaError_t launch_score_t(const ScoreParams& p, cudaStream_t st) {
  const size_t smem = score_smem_bytes(p.nb, D);
  auto kern = block_score_softmax_kernel<RT, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((p.nb + RT - 1) / RT, p.Hq, p.B);
  kern<<<grid, 256, smem, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_block_score_softmax(const ScoreParams& p, int D, cudaStream_t st) {
  const int RT = score_rows_per_cta(p.nb);
  if (RT == 16) return D == 128 ? launch_score_t<16, 128>(p, st) : launch_score_t<16, 64>(p, st);
  return D == 128 ? launch_score_t<8, 128>(p, st) : launch_score_t<8, 64>(p, st);
}

}  // namespace sfa
