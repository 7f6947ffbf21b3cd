// Exact attention over the kept key blocks ("Prism: Spectral-Aware
// Block-Sparse Attention" §1) on the sm_100a tensor cores.
//
// bf16 Q/K/V, query block = key block = 128 tokens, head dim 128.
// One CTA per (b, h, query block i); 6 warps:
//   warps 0-3  softmax: thread r owns query row r (TMEM lane r); reads S from
//              TMEM, online softmax in registers (lazy rescale of O), writes P
//              (bf16) into shared memory in the 128-byte-swizzled K-major
//              layout, final O / l epilogue.
//   warp 4     producer: TMA loads of the Q tile and of the K_j / V_j tiles of
//              every kept block j, fetched through the index list (two stages).
//   warp 5     MMA issuer: S = Q K_j^T (tcgen05.mma kind::f16, M=N=128,
//              K=16 steps) into a double-buffered TMEM S, then O += P V_j into
//              TMEM O; completion tracked with tcgen05.commit -> mbarriers.
// Every mbarrier wait is bounded (about 2 s); a wait that runs out writes
// SFA_ERR_TIMEOUT to the status word, raises a CTA-wide abort flag, drains
// the copies / MMAs this CTA issued and frees its tensor memory.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace sfa {

namespace {

constexpr int kHD = 128;
constexpr uint32_t kSub = 16384;       // 128 rows x 64 bf16 (one 128B-swizzle box)
constexpr uint32_t kTile = 2 * kSub;   // 128 x 128 bf16
constexpr int kStages = 2;
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + kTile;
constexpr uint32_t OFF_V = OFF_K + kStages * kTile;
constexpr uint32_t OFF_P = OFF_V + kStages * kTile;
constexpr uint32_t OFF_BAR = OFF_P + kTile;
enum { B_Q = 0, B_KF = 1, B_VF = 3, B_KVE = 5, B_SF = 7, B_SFREE = 9, B_PF = 11, B_OD = 12, B_DRAIN = 13, NBAR = 14 };
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;
constexpr int kThreads = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_O = 256;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8

struct Ctx {
  uint32_t sbase;
  volatile int* abort_flag;
  int* status;
  __device__ uint32_t bar(int k) const { return sbase + OFF_BAR + 8u * k; }
};

// Bounded wait on an mbarrier phase.  Returns false if the CTA aborted or the wait ran out.
__device__ bool wait_bar(const Ctx& c, uint32_t bar, uint32_t parity) {
  if (tc::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (tc::mbar_try_wait(bar, parity)) return true;
    if ((it & 127u) == 0) {
      if (*c.abort_flag) return false;
      if (globaltimer_ns() - t0 > kTimeoutNs) {
        *c.abort_flag = 1;
        report(c.status, SFA_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Bounded wait used while draining after an abort (ignores the abort flag).
__device__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!tc::mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kTimeoutNs) return;
  }
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, AttnParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  unsigned char* sm = smem_raw + pad;
  Ctx cx;
  cx.sbase = raw + pad;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  cx.abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);
  int* bad_flag = reinterpret_cast<int*>(sm + OFF_MISC + 8);
  cx.status = p.status;

  const int group = p.Hq / p.Hkv;
  int t = blockIdx.x;
  const int hh = t % group;
  t /= group;
  const int i = p.nb - 1 - (t % p.nb);
  t /= p.nb;
  const int g = t % p.Hkv;
  const int b = t / p.Hkv;
  const int h = g * group + hh;
  const size_t rowid = (size_t)(b * p.Hq + h) * p.nb + i;
  const int* list = p.idx + rowid * p.kmax;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (warp == 0) {
    // Validate the index list: count in [0, kmax], entries ascending in [0, nb), <= i if causal.
    const int n = p.counts[rowid];
    bool ok = n >= 0 && n <= p.kmax;
    if (ok) {
      for (int u = lane; u < n; u += 32) {
        const int j = list[u];
        if (j < 0 || j >= p.nb || (p.causal && j > i) || (u > 0 && list[u - 1] >= j)) ok = false;
      }
    }
    ok = __all_sync(0xffffffffu, ok);
    if (lane == 0) {
      *bad_flag = ok ? 0 : 1;
      if (!ok) report(p.status, SFA_ERR_INDEX);
      *cx.abort_flag = 0;
      tc::mbar_init(cx.bar(B_Q), 1);
      for (int s = 0; s < kStages; ++s) {
        tc::mbar_init(cx.bar(B_KF + s), 1);
        tc::mbar_init(cx.bar(B_VF + s), 1);
        tc::mbar_init(cx.bar(B_KVE + s), 1);
        tc::mbar_init(cx.bar(B_SF + s), 1);
        tc::mbar_init(cx.bar(B_SFREE + s), 128);
      }
      tc::mbar_init(cx.bar(B_PF), 128);
      tc::mbar_init(cx.bar(B_OD), 1);
      tc::mbar_init(cx.bar(B_DRAIN), 1);
      tc::fence_mbar_init();
    }
  } else if (warp == 4 && lane == 0) {
    tc::prefetch_tmap(&tmQ);
    tc::prefetch_tmap(&tmK);
    tc::prefetch_tmap(&tmV);
  } else if (warp == 5) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n = *bad_flag ? 0 : p.counts[rowid];
  const uint32_t sQ = cx.sbase + OFF_Q, sP = cx.sbase + OFF_P;

  if (n > 0 && warp == 4) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      const int qrow = (b * p.Hq + h) * p.L + i * 128;
      const int kvrow0 = (b * p.Hkv + g) * p.L;
      tc::mbar_arrive_expect_tx(cx.bar(B_Q), kTile);
      tc::tma_load_2d(sQ, &tmQ, cx.bar(B_Q), 0, qrow);
      tc::tma_load_2d(sQ + kSub, &tmQ, cx.bar(B_Q), 64, qrow);
      int issued[kStages] = {0, 0};
      for (int it = 0; it < n; ++it) {
        const int st = it & 1, use = it >> 1;
        if (!wait_bar(cx, cx.bar(B_KVE + st), (use & 1) ^ 1)) break;
        const int row = kvrow0 + list[it] * 128;
        const uint32_t sK = cx.sbase + OFF_K + st * kTile, sV = cx.sbase + OFF_V + st * kTile;
        tc::mbar_arrive_expect_tx(cx.bar(B_KF + st), kTile);
        tc::tma_load_2d(sK, &tmK, cx.bar(B_KF + st), 0, row);
        tc::tma_load_2d(sK + kSub, &tmK, cx.bar(B_KF + st), 64, row);
        tc::mbar_arrive_expect_tx(cx.bar(B_VF + st), kTile);
        tc::tma_load_2d(sV, &tmV, cx.bar(B_VF + st), 0, row);
        tc::tma_load_2d(sV + kSub, &tmV, cx.bar(B_VF + st), 64, row);
        issued[st] = use + 1;
      }
      if (*cx.abort_flag) {
        // Let every copy this CTA started land before the CTA exits.
        drain_wait(cx.bar(B_Q), 0);
        for (int s = 0; s < kStages; ++s) {
          if (issued[s] > 0) {
            drain_wait(cx.bar(B_KF + s), (issued[s] - 1) & 1);
            drain_wait(cx.bar(B_VF + s), (issued[s] - 1) & 1);
          }
        }
      }
    }
  } else if (n > 0 && warp == 5) {
    // ------------------------------ MMA issuer ----------------------------
    if (lane == 0) {
      const uint32_t id_qk = tc::idesc_bf16_f32(128, 128, false);
      const uint32_t id_pv = tc::idesc_bf16_f32(128, 128, true);
      if (wait_bar(cx, cx.bar(B_Q), 0)) {
        tc::tc_fence_after();
        for (int it = 0; it <= n; ++it) {
          if (it < n) {
            const int st = it & 1, use = it >> 1;
            if (!wait_bar(cx, cx.bar(B_KF + st), use & 1)) break;
            if (!wait_bar(cx, cx.bar(B_SFREE + st), (use & 1) ^ 1)) break;
            tc::tc_fence_after();
            const uint32_t sK = cx.sbase + OFF_K + st * kTile;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t off = (kk >> 2) * kSub + (kk & 3) * 32;
              tc::mma_bf16_ss(tmem + st * 128, tc::sw128_desc(sQ + off, 16, 1024),
                              tc::sw128_desc(sK + off, 16, 1024), id_qk, kk > 0 ? 1u : 0u);
            }
            tc::mma_commit(cx.bar(B_SF + st));
          }
          if (it >= 1) {
            const int jt = it - 1, st = jt & 1, use = jt >> 1;
            if (!wait_bar(cx, cx.bar(B_PF), jt & 1)) break;
            if (!wait_bar(cx, cx.bar(B_VF + st), use & 1)) break;
            tc::tc_fence_after();
            const uint32_t sV = cx.sbase + OFF_V + st * kTile;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t offp = (kk >> 2) * kSub + (kk & 3) * 32;
              tc::mma_bf16_ss(tmem + COL_O, tc::sw128_desc(sP + offp, 16, 1024),
                              tc::sw128_desc(sV + kk * 2048, kSub, 1024), id_pv,
                              (jt > 0 || kk > 0) ? 1u : 0u);
            }
            tc::mma_commit(cx.bar(B_KVE + st));
            tc::mma_commit(cx.bar(B_OD));
          }
        }
      }
      // All MMAs issued by this thread complete before teardown.
      tc::mma_commit(cx.bar(B_DRAIN));
      drain_wait(cx.bar(B_DRAIN), 0);
    }
  } else if (n > 0 && warp < 4) {
    // ------------------------------ softmax -------------------------------
    const int r = threadIdx.x;
    const int qt = i * 128 + r;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const float sl2 = p.scale * 1.4426950408889634f;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    unsigned char* prow = sm + OFF_P + r * 128;
    for (int it = 0; it < n; ++it) {
      const int sb = it & 1, use = it >> 1;
      ok = __all_sync(0xffffffffu, wait_bar(cx, cx.bar(B_SF + sb), use & 1));
      if (!ok) break;
      tc::tc_fence_after();
      float x[128];
      {
        uint32_t v[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          tc::tmem_ld32(tmem + lane_base + sb * 128 + c * 32, v);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) x[c * 32 + e] = __uint_as_float(v[e]);
        }
      }
      tc::tc_fence_before();
      tc::mbar_arrive(cx.bar(B_SFREE + sb));
      const int j = list[it];
      const int lim = (p.causal && j * 128 + 127 > qt) ? qt - j * 128 : 127;  // keys c <= lim visible
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        const float v = (c <= lim) ? x[c] * sl2 : -INFINITY;
        x[c] = v;
        mx = fmaxf(mx, v);
      }
      const float mnew = fmaxf(m, mx);
      if (it > 0) {
        ok = __all_sync(0xffffffffu, wait_bar(cx, cx.bar(B_OD), (it - 1) & 1));
        if (!ok) break;
      }
      const bool need = mnew > m + kRescaleThreshold || (m == -INFINITY && mnew != -INFINITY);
      if (__any_sync(0xffffffffu, need)) {
        const float f = need ? exp2f(m - mnew) : 1.f;
        if (it > 0) {
          tc::tc_fence_after();
          uint32_t v[32];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint32_t ta = tmem + lane_base + COL_O + c * 32;
            tc::tmem_ld32(ta, v);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * f);
            tc::tmem_st32(ta, v);
          }
          tc::tmem_wait_st();
        }
        if (need) {
          l *= f;
          m = mnew;
        }
      }
      const float mu = (m == -INFINITY) ? 0.f : m;
      float rs = 0.f;
#pragma unroll
      for (int cc = 0; cc < 16; ++cc) {
        float pv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          pv[e] = exp2f(x[cc * 8 + e] - mu);
          rs += pv[e];
        }
        uint4 u;
        u.x = pack_bf16x2(pv[0], pv[1]);
        u.y = pack_bf16x2(pv[2], pv[3]);
        u.z = pack_bf16x2(pv[4], pv[5]);
        u.w = pack_bf16x2(pv[6], pv[7]);
        const int sub = cc >> 3, ch = cc & 7;
        *reinterpret_cast<uint4*>(prow + sub * kSub + ((ch ^ (r & 7)) << 4)) = u;
      }
      l += rs;
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      tc::mbar_arrive(cx.bar(B_PF));
    }
    if (ok) ok = __all_sync(0xffffffffu, wait_bar(cx, cx.bar(B_OD), (n - 1) & 1));
    if (ok) {
      tc::tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.O) + ((size_t)(b * p.Hq + h) * p.L + qt) * kHD;
      uint32_t v[32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        tc::tmem_ld32(tmem + lane_base + COL_O + c * 32, v);
        tc::tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 u;
          u.x = pack_bf16x2(__uint_as_float(v[q * 8 + 0]) * inv, __uint_as_float(v[q * 8 + 1]) * inv);
          u.y = pack_bf16x2(__uint_as_float(v[q * 8 + 2]) * inv, __uint_as_float(v[q * 8 + 3]) * inv);
          u.z = pack_bf16x2(__uint_as_float(v[q * 8 + 4]) * inv, __uint_as_float(v[q * 8 + 5]) * inv);
          u.w = pack_bf16x2(__uint_as_float(v[q * 8 + 6]) * inv, __uint_as_float(v[q * 8 + 7]) * inv);
          *reinterpret_cast<uint4*>(orow + c * 32 + q * 8) = u;
        }
      }
      if (p.lse != nullptr)
        p.lse[(size_t)(b * p.Hq + h) * p.L + qt] = l > 0.f ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
    }
  }
  if (n == 0 && warp < 4) {
    const int qt = i * 128 + threadIdx.x;
    uint4* orow = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.O) +
                                           ((size_t)(b * p.Hq + h) * p.L + qt) * kHD);
#pragma unroll
    for (int q = 0; q < 16; ++q) orow[q] = make_uint4(0, 0, 0, 0);
    if (p.lse != nullptr) p.lse[(size_t)(b * p.Hq + h) * p.L + qt] = -INFINITY;
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

cudaError_t launch_attn_tcgen05(const AttnParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                const CUtensorMap& tmV, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)((size_t)p.B * p.Hq * p.nb);
  attn_tc_kernel<<<grid, kThreads, SMEM_BYTES, st>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

}  // namespace sfa
