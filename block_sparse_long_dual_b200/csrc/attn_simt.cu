// Exact attention over the kept key blocks ("Prism: Spectral-Aware
// Block-Sparse Attention" §1) on the float32 CUDA cores.
//
// This kernel serves the shapes the tcgen05 kernel does not take (float32
// tensors, block 64, head dim 64): it computes in float32 throughout, which the
// 1e-4 float32 tolerance needs (TF32 tensor cores could not meet it).
// CTA = one query block (BLK rows) of one (b, h); 4 threads per query row, each
// owning D/4 dims of q and of the output accumulator; K_j / V_j tiles of every
// kept block staged in shared memory as float32; online softmax in chunks of
// 16 keys.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace sfa {

template <typename T, int D, int BLK>
__global__ void __launch_bounds__(BLK * 4) attn_simt_kernel(AttnParams p) {
  constexpr int DP = D / 4;        // dims per thread
  constexpr int LD = D + 4;        // padded smem row (floats)
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* Ks = reinterpret_cast<float*>(smem_raw);
  float* Vs = Ks + BLK * LD;
  __shared__ int bad;

  const int tile = blockIdx.x;
  const int i = tile % p.nb;
  const int h = (tile / p.nb) % p.Hq;
  const int b = tile / (p.nb * p.Hq);
  const int g = h / (p.Hq / p.Hkv);
  const int tid = threadIdx.x;
  const int r = tid >> 2, part = tid & 3;
  const size_t qrow = ((size_t)(b * p.Hq + h) * p.L) + (size_t)i * BLK + r;
  const size_t kvbase = (size_t)(b * p.Hkv + g) * p.L;
  const size_t rowid = (size_t)(b * p.Hq + h) * p.nb + i;
  const int* list = p.idx + rowid * p.kmax;

  // Validate the index list once (ascending, in range, causal).
  if (tid == 0) {
    int ok = 1;
    const int n = p.counts[rowid];
    if (n < 0 || n > p.kmax) ok = 0;
    for (int t = 0; ok && t < n; ++t) {
      const int j = list[t];
      if (j < 0 || j >= p.nb || (t > 0 && j <= list[t - 1]) || (p.causal && j > i)) ok = 0;
    }
    bad = !ok;
    if (!ok) report(p.status, SFA_ERR_INDEX);
  }
  __syncthreads();
  const int n = bad ? 0 : p.counts[rowid];

  float q[DP], o[DP];
  {
    const T* qp = static_cast<const T*>(p.Q) + qrow * D + part * DP;
    // RoPE on load: dims [part DP, +DP) pair with the other half's dims (+-d/2).
    const bool rot = p.rope_cos != nullptr;
    const bool upper = part >= 2;
    const T* pp = static_cast<const T*>(p.Q) + qrow * D + (part ^ 2) * DP;
    const size_t tpos = (size_t)i * BLK + r;
    const int m0 = (part & 1) * DP;  // first rotary pair index of this thread's dims
#pragma unroll
    for (int d = 0; d < DP; d += 8) {
      float v[8];
      load8(qp + d, v);
      if (rot) {
        float w[8], c[8], sn[8];
        load8(pp + d, w);
        load8(p.rope_cos + tpos * (D / 2) + m0 + d, c);
        load8(p.rope_sin + tpos * (D / 2) + m0 + d, sn);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float lo, hi;
          if (upper) rope_pair(w[e], v[e], c[e], sn[e], lo, hi); else rope_pair(v[e], w[e], c[e], sn[e], lo, hi);
          v[e] = round_as(upper ? hi : lo, T());
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) { q[d + e] = v[e] * p.scale; o[d + e] = 0.f; }
    }
  }
  float m = -INFINITY, l = 0.f;
  const int qt = i * BLK + r;

  for (int it = 0; it < n; ++it) {
    const int j = list[it];
    __syncthreads();
    const T* kp = static_cast<const T*>(p.K) + (kvbase + (size_t)j * BLK) * D;
    const T* vp = static_cast<const T*>(p.V) + (kvbase + (size_t)j * BLK) * D;
    for (int e = tid * 8; e < BLK * D; e += BLK * 4 * 8) {
      const int rr = e / D, cc = e % D;
      float v[8];
      load8(kp + e, v);
#pragma unroll
      for (int u = 0; u < 8; ++u) Ks[rr * LD + cc + u] = v[u];
      load8(vp + e, v);
#pragma unroll
      for (int u = 0; u < 8; ++u) Vs[rr * LD + cc + u] = v[u];
    }
    __syncthreads();
    for (int s0 = 0; s0 < BLK; s0 += 16) {
      float sc[16];
      float cmax = -INFINITY;
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const float* kr = Ks + (s0 + u) * LD + part * DP;
        float acc = 0.f;
#pragma unroll
        for (int d = 0; d < DP; d += 4) {
          const float4 k4 = *reinterpret_cast<const float4*>(kr + d);
          acc = fmaf(q[d], k4.x, acc);
          acc = fmaf(q[d + 1], k4.y, acc);
          acc = fmaf(q[d + 2], k4.z, acc);
          acc = fmaf(q[d + 3], k4.w, acc);
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        const int kt = j * BLK + s0 + u;
        if (p.causal && kt > qt) acc = -INFINITY;
        sc[u] = acc;
        cmax = fmaxf(cmax, acc);
      }
      const float mnew = fmaxf(m, cmax);
      if (mnew == -INFINITY) continue;
      const float corr = expf(m - mnew);  // m = -inf gives 0
      l *= corr;
#pragma unroll
      for (int d = 0; d < DP; ++d) o[d] *= corr;
      m = mnew;
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const float pr = expf(sc[u] - m);
        l += pr;
        const float* vr = Vs + (s0 + u) * LD + part * DP;
#pragma unroll
        for (int d = 0; d < DP; d += 4) {
          const float4 v4 = *reinterpret_cast<const float4*>(vr + d);
          o[d] = fmaf(pr, v4.x, o[d]);
          o[d + 1] = fmaf(pr, v4.y, o[d + 1]);
          o[d + 2] = fmaf(pr, v4.z, o[d + 2]);
          o[d + 3] = fmaf(pr, v4.w, o[d + 3]);
        }
      }
    }
  }

  const float inv = l > 0.f ? 1.f / l : 0.f;
  T* op = static_cast<T*>(p.O) + qrow * D + part * DP;
#pragma unroll
  for (int d = 0; d < DP; d += 8) {
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = o[d + e] * inv;
    store8(op + d, v);
  }
  if (p.lse != nullptr && part == 0) p.lse[qrow] = l > 0.f ? m + logf(l) : -INFINITY;
}

template <typename T, int D, int BLK>
static cudaError_t launch_simt_t(const AttnParams& p, cudaStream_t st) {
  const size_t smem = (size_t)2 * BLK * (D + 4) * sizeof(float);
  auto kern = attn_simt_kernel<T, D, BLK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)((size_t)p.B * p.Hq * p.nb);
  kern<<<grid, BLK * 4, smem, st>>>(p);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_simt_dt(const AttnParams& p, int D, cudaStream_t st) {
  if (D == 64) return p.block == 64 ? launch_simt_t<T, 64, 64>(p, st) : launch_simt_t<T, 64, 128>(p, st);
  return p.block == 64 ? launch_simt_t<T, 128, 64>(p, st) : launch_simt_t<T, 128, 128>(p, st);
}

cudaError_t launch_attn_simt(const AttnParams& p, int dtype, int D, cudaStream_t st) {
  if (dtype == SFA_BF16) return launch_simt_dt<__nv_bfloat16>(p, D, st);
  return launch_simt_dt<float>(p, D, st);
}

}  // namespace sfa
