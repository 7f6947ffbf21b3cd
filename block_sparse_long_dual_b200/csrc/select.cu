// Per-query-block selection of key blocks ("Prism: Spectral-Aware
// Block-Sparse Attention" §1: attention runs over a chosen subset of blocks).
//
// One CTA per row (b, h, i).  The candidates {0..i} minus the forced blocks
// are sorted in shared memory by a bitonic network on (probability desc,
// index asc); top-k takes a prefix of fixed length, cumulative mass takes the
// shortest prefix whose float64 running sum (forced blocks included) reaches
// `mass`.  The kept set is written ascending, padded with -1.
#include "common.cuh"
#include "kernels.h"

namespace sfa {

namespace {

__device__ __forceinline__ bool before(float ka, int ia, float kb, int ib) {
  return ka > kb || (ka == kb && ia < ib);
}

// Exclusive block scan of one value per thread (256 threads).
template <typename V>
__device__ V block_exclusive_scan(V v, V* warp_tot, V* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  V inc = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const V n = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += n;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  V base = 0, all = 0;
  for (int w = 0; w < 8; ++w) {
    if (w < warp) base += warp_tot[w];
    all += warp_tot[w];
  }
  if (total) *total = all;
  __syncthreads();
  return base + inc - v;
}

}  // namespace

__global__ void __launch_bounds__(256) select_kernel(SelectParams p, int nb2) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* key = reinterpret_cast<float*>(smem_raw);
  int* id = reinterpret_cast<int*>(key + nb2);
  unsigned char* flag = reinterpret_cast<unsigned char*>(id + nb2);
  __shared__ double dtot[8];
  __shared__ int itot[8];

  const int row = blockIdx.x;
  const int i = row % p.nb;
  const float* prow = p.probs + (size_t)row * p.nb;
  const int tid = threadIdx.x;
  int S = 1;
  while (S < i + 1) S <<= 1;
  const int f0 = i;
  const int f1 = ((p.flags & SFA_KEEP_SINK) && i > 0) ? 0 : -1;
  const int nforced = f1 >= 0 ? 2 : 1;
  const int nc = i + 1 - nforced;

  for (int t = tid; t < S; t += 256) {
    if (t <= i) {
      const bool forced = (t == f0) || (t == f1);
      key[t] = forced ? -1.f : prow[t];
    } else {
      key[t] = -2.f;
    }
    id[t] = t;
  }
  for (int t = tid; t < p.nb; t += 256) flag[t] = 0;
  __syncthreads();

  for (int k2 = 2; k2 <= S; k2 <<= 1) {
    for (int j2 = k2 >> 1; j2 > 0; j2 >>= 1) {
      for (int t = tid; t < (S >> 1); t += 256) {
        const int a = 2 * j2 * (t / j2) + (t % j2);
        const int c = a + j2;
        const bool up = (a & k2) == 0;
        const float ka = key[a], kc = key[c];
        const int ia = id[a], ic = id[c];
        const bool sw = up ? before(kc, ic, ka, ia) : before(ka, ia, kc, ic);
        if (sw) {
          key[a] = kc; key[c] = ka;
          id[a] = ic; id[c] = ia;
        }
      }
      __syncthreads();
    }
  }

  int ntake;
  if (p.k >= 0) {
    ntake = min(p.k, nc);
  } else {
    double cum_forced = (double)prow[f0] + (f1 >= 0 ? (double)prow[f1] : 0.0);
    const int ept = (S + 255) / 256;
    const int t0 = tid * ept;
    double local = 0.0;
    for (int t = t0; t < min(t0 + ept, nc); ++t) local += (double)key[t];
    double excl = block_exclusive_scan<double>(local, dtot, nullptr);
    double run = cum_forced + excl;
    int cnt = 0;
    for (int t = t0; t < min(t0 + ept, nc); ++t) {
      if (run < p.mass) ++cnt;
      run += (double)key[t];
    }
    int total = 0;
    block_exclusive_scan<int>(cnt, itot, &total);
    ntake = total;
  }
  for (int t = tid; t < ntake; t += 256) flag[id[t]] = 1;
  if (tid == 0) {
    flag[f0] = 1;
    if (f1 >= 0) flag[f1] = 1;
  }
  __syncthreads();

  // Ascending compaction of the kept flags over [0, i].
  const int n = i + 1;
  const int ept = (n + 255) / 256;
  const int t0 = tid * ept;
  int cnt = 0;
  for (int t = t0; t < min(t0 + ept, n); ++t) cnt += flag[t];
  int total = 0;
  int pos = block_exclusive_scan<int>(cnt, itot, &total);
  int* out = p.idx + (size_t)row * p.kmax;
  for (int t = t0; t < min(t0 + ept, n); ++t)
    if (flag[t]) out[pos++] = t;
  for (int t = total + tid; t < p.kmax; t += 256) out[t] = -1;
  if (tid == 0) p.counts[row] = total;
}

cudaError_t launch_select(const SelectParams& p, cudaStream_t st) {
  int nb2 = 1;
  while (nb2 < p.nb) nb2 <<= 1;
  const size_t smem = (size_t)nb2 * (sizeof(float) + sizeof(int)) + (size_t)p.nb;
  const unsigned grid = (unsigned)((size_t)p.B * p.Hq * p.nb);
  select_kernel<<<grid, 256, smem, st>>>(p, nb2);
  return cudaGetLastError();
}

}  // namespace sfa
