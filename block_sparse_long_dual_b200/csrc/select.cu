// Per-query-block selection of key blocks ("Prism: Spectral-Aware
// Block-Sparse Attention" §1): one warp per row (b, h, i) running the shared
// warp routine of select_row.cuh on the row's float32 probabilities.
#include "common.cuh"
#include "kernels.h"
#include "select_row.cuh"

namespace sfa {

namespace {

constexpr int kWarps = 8;

template <int NPL>
__global__ void __launch_bounds__(kWarps * 32) select_kernel(SelectParams p) {
  const int lane = threadIdx.x & 31;
  const size_t row = (size_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const size_t nrows = (size_t)p.B * p.Hq * p.nb;
  if (row >= nrows) return;
  const int i = (int)(row % p.nb);
  const float* prow = p.probs + row * p.nb;
  auto prob = [&](int j) { return __ldg(prow + j); };
  int* out = p.idx + row * p.kmax;
  // A row's causal prefix (blocks 0 .. i) fills i / 32 + 1 register slots: rows in the first
  // quarter (half) of the range run the routine with a quarter (half) of the slots, so their
  // bisection steps scan only those.
  int n;
  if (NPL >= 16 && i < NPL * 8)
    n = select_row_warp<(NPL >= 16 ? NPL / 4 : 1)>(prob, i, p.k, p.mass, p.flags, out, p.kmax);
  else if (NPL >= 16 && i < NPL * 16)
    n = select_row_warp<(NPL >= 16 ? NPL / 2 : 1)>(prob, i, p.k, p.mass, p.flags, out, p.kmax);
  else
    n = select_row_warp<NPL>(prob, i, p.k, p.mass, p.flags, out, p.kmax);
  if (lane == 0) p.counts[row] = n;
}

template <int NPL>
cudaError_t launch_t(const SelectParams& p, cudaStream_t st) {
  const size_t rows = (size_t)p.B * p.Hq * p.nb;
  const unsigned grid = (unsigned)((rows + kWarps - 1) / kWarps);
  select_kernel<NPL><<<grid, kWarps * 32, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select(const SelectParams& p, cudaStream_t st) {
  if (p.nb <= 32) return launch_t<1>(p, st);
  if (p.nb <= 64) return launch_t<2>(p, st);
  if (p.nb <= 128) return launch_t<4>(p, st);
  if (p.nb <= 256) return launch_t<8>(p, st);
  if (p.nb <= 512) return launch_t<16>(p, st);
  if (p.nb <= 1024) return launch_t<32>(p, st);
  return launch_t<64>(p, st);
}

}  // namespace sfa
