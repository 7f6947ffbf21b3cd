// Exact attention over the kept key blocks ("Prism: Spectral-Aware
// Block-Sparse Attention" §1) on the sm_100a tensor cores.
//
// bf16 Q/K/V, query block = key block = 128 tokens, head dim 128.
// A CTA holds KT query tiles (Layout<KT>): consecutive entries of the tile order
// (b, kv head, query block descending, q head in the group).  With KT = 2 (long
// index lists) the two tiles, two Q heads of one GQA group at the same query
// block, ping-pong on the tensor core: while one softmax warpgroup turns S_t
// into P_t, the tensor core runs the other tile's P.V and next Q.K^T.  With
// KT = 1 (short lists) two CTAs share each SM and play the same game, and one
// CTA's prologue (barriers, tensor memory, Q) and epilogue (O) hide behind the
// other's main loop.
//
//   warps 0 .. 4 KT - 1  softmax of tile w / 4: one thread per query row r
//                    (TMEM lane r = 32 (w % 4) + lane).  The thread loads its
//                    whole row of S_t (128 columns) into registers, takes the
//                    row maximum with no exchange, rescales O_t lazily, computes
//                    P_t from the same registers and writes it (bf16) back into
//                    the S_t columns of TMEM; final O_t / l epilogue.
//   warp 4 KT        producer: TMA loads of Q_t (started at entry, while warps 0
//                    and 4 validate the index lists) and of K_t(j), V_t(j) for
//                    every kept block j of each tile (one K and one V slot per tile).
//   warp 4 KT + 1    MMA issuer: S_t = Q_t K_t^T (A, B from shared memory) and
//                    O_t += P_t V_t (A = P_t from TMEM, B = V_t from shared
//                    memory), M = N = 128, K = 16 steps; completion tracked with
//                    tcgen05.commit -> mbarriers.  A commit covers every MMA the
//                    thread issued before it, so the commit that signals S_t(j)
//                    also means O_t has absorbed P_t(j-1).  The softmax threads
//                    signal P_t in two parts (keys [0, 64), then [64, 128)), so
//                    half of P_t.V_t runs while they compute the rest.
// TMEM (256 KT columns): S_t at [128 t, 128 t + 128), O_t at [128 (KT + t), +128);
// P_t aliases S_t (two bf16 per column): keys [16 c, 16 c + 16) in S columns
// [8 c, 8 c + 8), written once the whole row of S_t is in registers.
// Every mbarrier wait is bounded (about 2 s); a wait that runs out writes
// SFA_ERR_TIMEOUT to the status word, raises a CTA-wide abort flag, drains the
// copies / MMAs this CTA issued and frees its tensor memory.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace sfa {

namespace {

constexpr int kHD = 128;
constexpr uint32_t kSub = 16384;       // 128 rows x 64 bf16 (one 128B-swizzle box)
constexpr uint32_t kTile = 2 * kSub;   // 128 x 128 bf16
// Barriers, two of each (one per tile) except DRAIN and QR.
enum { B_Q = 0, B_KF = 2, B_VF = 4, B_KE = 6, B_VE = 8, B_SF = 10, B_PF = 12, B_OD = 14, B_PH = 16, B_DRAIN = 18,
       B_QR = 19, NBAR = 20 };  // B_PH: the first half of P_t written (B_PF: all of it); B_QR: the CTA's
                                // Q tiles rotated in shared memory (RoPE on load)
constexpr int kMaxList = 2048;  // nb <= 2048, so a valid list has <= 2048 entries
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8

// Layout for KT query tiles per CTA.  KT = 2: one CTA ping-pongs two tiles on the tensor core;
// KT = 1: half the shared memory and tensor memory, so two CTAs share an SM and each one's
// prologue and epilogue overlap the other's main loop (better when the index lists are short).
template <int KT>
struct Layout {
  static_assert(KT == 1 || KT == 2, "one or two query tiles per CTA");
  // Shared memory: per tile t a Q, a K and a V tile (3 KT x 32 KB), barriers, exchange, lists.
  static __host__ __device__ constexpr uint32_t off_q(int t) { return t * kTile; }
  static __host__ __device__ constexpr uint32_t off_k(int t) { return KT * kTile + t * kTile; }
  static __host__ __device__ constexpr uint32_t off_v(int t) { return 2 * KT * kTile + t * kTile; }
  static constexpr uint32_t OFF_BAR = 3 * KT * kTile;
  static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr uint32_t OFF_LIST = OFF_MISC + 32;  // per tile: the validated index list
  static constexpr uint32_t SMEM_BYTES = OFF_LIST + KT * kMaxList * 4 + 1024;
  // Warps 0 .. 4 KT - 1: softmax of tile w / 4 (one thread per query row, warp w on TMEM lanes
  // [32 (w % 4), +32)); then the TMA producer and the MMA issuer.
  static constexpr int kSoftmaxThreads = KT * 128;
  static constexpr int kThreads = kSoftmaxThreads + 64;
  static constexpr int kProducerWarp = KT * 4, kMmaWarp = KT * 4 + 1;
  static constexpr uint32_t TMEM_COLS = KT * 256;
  static __host__ __device__ constexpr uint32_t col_s(int t) { return t * 128; }
  static __host__ __device__ constexpr uint32_t col_o(int t) { return KT * 128 + t * 128; }
};

struct Ctx {
  uint32_t sbase;
  uint32_t bars;  // shared address of barrier 0
  volatile int* abort_flag;
  int* status;
  __device__ uint32_t bar(int k) const { return bars + 8u * k; }
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

struct Tile {
  int b, h, g, i, n;
  const int* list;
  bool valid;
};

__device__ Tile decode_tile(const AttnParams& p, int t) {
  Tile x;
  const int group = p.Hq / p.Hkv;
  const int total = p.B * p.Hq * p.nb;
  x.valid = t < total;
  if (!x.valid) t = total - 1;
  const int hh = t % group;
  t /= group;
  x.i = p.nb - 1 - (t % p.nb);
  t /= p.nb;
  x.g = t % p.Hkv;
  x.b = t / p.Hkv;
  x.h = x.g * group + hh;
  x.list = p.idx + ((size_t)(x.b * p.Hq + x.h) * p.nb + x.i) * p.kmax;
  x.n = 0;
  return x;
}

// RoPE on load: the 128 KT softmax threads rotate the CTA's Q tiles in shared
// memory once their TMA copies have landed (bounded waits on the tiles' B_Q
// barriers); returns false if a wait gave up.  Work unit = (row, 16-byte
// chunk c) of a tile: chunk c of box 0 holds dims [8c, 8c + 8) and the same
// offset of box 1 holds their rotary partners [64 + 8c, 64 + 8c + 8) (chunk c of
// row r is stored at chunk c ^ (r & 7) of the 128-byte row).  Thread st takes
// chunk st & 7 of rows st / 8 + 16 KT k (k < 8 / KT), so a warp touches four
// whole rows: conflict-free in shared memory, and each row's table entries are
// one contiguous 256-byte run.  Rows go four at a time; the first four rows'
// table entries are fetched before the waits, so their latency hides behind
// the copies.  The two tiles usually share the query block (two heads of a GQA
// group): the entries then serve both.  Kept out of line: it runs once per CTA
// and must not add to the register pressure of the softmax loop.
template <int KT>
__device__ __noinline__ bool rope_q_on_load(volatile int* abort_flag, int* status, uint32_t bar_q0,
                                            unsigned char* sm, const float* cos_t, const float* sin_t, int i0,
                                            int i1, int n0, int n1, int st) {
  Ctx cx;
  cx.sbase = 0;
  cx.bars = 0;
  cx.abort_flag = abort_flag;
  cx.status = status;
  constexpr int RS = 16 * KT, RPT = 128 / RS, GR = 4;  // row stride, rows per thread, rows per group
  static_assert(RPT % GR == 0, "whole groups of rows");
  const int c = st & 7;
  const bool two = KT == 2 && n0 > 0 && n1 > 0 && i1 != i0;  // tiles at different query blocks: two slices
  const int ia = n0 > 0 ? i0 : i1;
#pragma unroll 1
  for (int g0 = 0; g0 < RPT; g0 += GR) {
    float ca[GR][8], sa[GR][8], cb[GR][8], sb[GR][8];
#pragma unroll
    for (int k = 0; k < GR; ++k) {
      const int row = (st >> 3) + RS * (g0 + k);
      load8(cos_t + ((size_t)ia * 128 + row) * 64 + c * 8, ca[k]);
      load8(sin_t + ((size_t)ia * 128 + row) * 64 + c * 8, sa[k]);
      if (two) {
        load8(cos_t + ((size_t)i1 * 128 + row) * 64 + c * 8, cb[k]);
        load8(sin_t + ((size_t)i1 * 128 + row) * 64 + c * 8, sb[k]);
      }
    }
    if (g0 == 0) {
      bool ok = true;
      if (n0 > 0) ok = wait_bar(cx, bar_q0, 0);
      if (ok && KT == 2 && n1 > 0) ok = wait_bar(cx, bar_q0 + 8, 0);  // B_Q + 1
      if (!__all_sync(0xffffffffu, ok)) return false;
    }
#pragma unroll
    for (int t = 0; t < KT; ++t) {
      if ((t == 0 ? n0 : n1) == 0) continue;
      const bool use_b = t == 1 && two;
#pragma unroll
      for (int k = 0; k < GR; ++k) {
        const int row = (st >> 3) + RS * (g0 + k);
        unsigned char* rp = sm + Layout<KT>::off_q(t) + row * 128 + ((c ^ (row & 7)) << 4);
        uint4* plo = reinterpret_cast<uint4*>(rp);
        uint4* phi = reinterpret_cast<uint4*>(rp + kSub);
        const uint4 ulo = *plo, uhi = *phi;
        const uint32_t wl[4] = {ulo.x, ulo.y, ulo.z, ulo.w}, wh[4] = {uhi.x, uhi.y, uhi.z, uhi.w};
        uint32_t ol[4], oh[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float c0 = use_b ? cb[k][2 * e] : ca[k][2 * e], s0 = use_b ? sb[k][2 * e] : sa[k][2 * e];
          const float c1 = use_b ? cb[k][2 * e + 1] : ca[k][2 * e + 1];
          const float s1 = use_b ? sb[k][2 * e + 1] : sa[k][2 * e + 1];
          float l0, l1, h0, h1;
          rope_pair(__uint_as_float(wl[e] << 16), __uint_as_float(wh[e] << 16), c0, s0, l0, h0);
          rope_pair(__uint_as_float(wl[e] & 0xFFFF0000u), __uint_as_float(wh[e] & 0xFFFF0000u), c1, s1, l1, h1);
          ol[e] = pack_bf16x2(l0, l1);
          oh[e] = pack_bf16x2(h0, h1);
        }
        *plo = make_uint4(ol[0], ol[1], ol[2], ol[3]);
        *phi = make_uint4(oh[0], oh[1], oh[2], oh[3]);
      }
    }
  }
  tc::fence_proxy_async_smem();  // the generic-proxy writes become visible to the MMAs
  return true;
}

}  // namespace

template <int KT>
__global__ void __launch_bounds__(Layout<KT>::kThreads, 3 - KT)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, AttnParams p) {
  using L = Layout<KT>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  unsigned char* sm = smem_raw + pad;
  Ctx cx;
  cx.sbase = raw + pad;
  cx.bars = cx.sbase + L::OFF_BAR;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::OFF_MISC);
  cx.abort_flag = reinterpret_cast<volatile int*>(sm + L::OFF_MISC + 4);
  int* nsh = reinterpret_cast<int*>(sm + L::OFF_MISC + 8);  // validated count per tile
  int* slist = reinterpret_cast<int*>(sm + L::OFF_LIST);    // [KT][kMaxList] validated index lists
  cx.status = p.status;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  Tile tl[2];
  tl[0] = decode_tile(p, KT * blockIdx.x);
  tl[1] = decode_tile(p, KT == 2 ? 2 * blockIdx.x + 1 : KT * blockIdx.x);
  if (KT == 1) tl[1].valid = false;
  bool qearly[2] = {false, false};  // producer: Q copy started before the lists were validated

  if (warp == 0 || (KT == 2 && warp == 4)) {
    // Validate one tile's index list: count in [0, kmax], entries ascending in [0, nb), <= i if causal.
    const int t = warp >> 2;
    const Tile x = t == 0 ? tl[0] : tl[1];
    int n = 0;
    if (x.valid) {
      const size_t rowid = (size_t)(x.b * p.Hq + x.h) * p.nb + x.i;
      // The count and the list's first 32 slots are loaded together (a row holds kmax slots), so a
      // list of up to 32 entries costs one round trip; each entry is compared with its predecessor
      // through a shuffle.
      int j0 = lane < p.kmax ? x.list[lane] : 0;
      n = p.counts[rowid];
      bool ok = n >= 0 && n <= p.kmax;
      if (ok) {
        int prev = -1;  // last entry of the previous 32
        for (int u0 = 0; u0 < n; u0 += 32) {
          const int u = u0 + lane;
          const int j = u0 == 0 ? j0 : (u < n ? x.list[u] : 0);
          const int up = __shfl_up_sync(0xffffffffu, j, 1);
          const int before = lane == 0 ? prev : up;
          if (u < n) {
            if (j < 0 || j >= p.nb || (p.causal && j > x.i) || (u > 0 && before >= j)) ok = false;
            if (u < kMaxList) slist[t * kMaxList + u] = j;
          }
          prev = __shfl_sync(0xffffffffu, j, 31);
        }
      }
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0) report(p.status, SFA_ERR_INDEX);
        n = 0;
      }
    }
    if (lane == 0) nsh[t] = n;
  } else if (warp == L::kProducerWarp && lane == 0) {
    *cx.abort_flag = 0;
    for (int k = 0; k < NBAR; ++k)
      tc::mbar_init(cx.bar(k), k == B_QR ? L::kSoftmaxThreads
                               : (k == B_PF || k == B_PF + 1 || k == B_PH || k == B_PH + 1) ? 128 : 1);
    tc::fence_mbar_init();
    tc::prefetch_tmap(&tmQ);
    tc::prefetch_tmap(&tmK);
    tc::prefetch_tmap(&tmV);
    // A Q tile depends only on the tile, not on its list: its copy starts while the lists are
    // being validated.
#pragma unroll
    for (int t = 0; t < KT; ++t) {
      if (!tl[t].valid) continue;
      const int qrow = (tl[t].b * p.Hq + tl[t].h) * p.L + tl[t].i * 128;
      const uint32_t sQ = cx.sbase + L::off_q(t);
      tc::mbar_arrive_expect_tx(cx.bar(B_Q + t), kTile);
      tc::tma_load_2d(sQ, &tmQ, cx.bar(B_Q + t), 0, qrow);
      tc::tma_load_2d(sQ + kSub, &tmQ, cx.bar(B_Q + t), 64, qrow);
      qearly[t] = true;
    }
  } else if (warp == L::kMmaWarp) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), L::TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  tl[0].n = nsh[0];
  tl[1].n = KT == 2 ? nsh[1] : 0;
  const int nmax = max(tl[0].n, tl[1].n);

  if (warp == L::kProducerWarp) {
    // ------------------------------ producer ------------------------------
    if (lane == 0 && nmax > 0) {
      int kissued[2] = {0, 0}, vissued[2] = {0, 0};
      bool ok = true;
      for (int it = 0; ok && it < nmax; ++it) {
#pragma unroll
        for (int t = 0; t < KT; ++t) {
          if (!ok || it >= tl[t].n) continue;
          if (it > 0 && !wait_bar(cx, cx.bar(B_KE + t), (it - 1) & 1)) { ok = false; break; }
          const int row = (tl[t].b * p.Hkv + tl[t].g) * p.L + slist[t * kMaxList + it] * 128;
          const uint32_t sK = cx.sbase + L::off_k(t);
          tc::mbar_arrive_expect_tx(cx.bar(B_KF + t), kTile);
          tc::tma_load_2d(sK, &tmK, cx.bar(B_KF + t), 0, row);
          tc::tma_load_2d(sK + kSub, &tmK, cx.bar(B_KF + t), 64, row);
          kissued[t] = it + 1;
        }
#pragma unroll
        for (int t = 0; t < KT; ++t) {
          if (!ok || it >= tl[t].n) continue;
          if (it > 0 && !wait_bar(cx, cx.bar(B_VE + t), (it - 1) & 1)) { ok = false; break; }
          const int row = (tl[t].b * p.Hkv + tl[t].g) * p.L + slist[t * kMaxList + it] * 128;
          const uint32_t sV = cx.sbase + L::off_v(t);
          tc::mbar_arrive_expect_tx(cx.bar(B_VF + t), kTile);
          tc::tma_load_2d(sV, &tmV, cx.bar(B_VF + t), 0, row);
          tc::tma_load_2d(sV + kSub, &tmV, cx.bar(B_VF + t), 64, row);
          vissued[t] = it + 1;
        }
      }
      if (*cx.abort_flag) {
        // Let every copy this CTA started land before the CTA exits.
        for (int t = 0; t < KT; ++t) {
          if (kissued[t] > 0) drain_wait(cx.bar(B_KF + t), (kissued[t] - 1) & 1);
          if (vissued[t] > 0) drain_wait(cx.bar(B_VF + t), (vissued[t] - 1) & 1);
        }
      }
    }
    // Every Q copy lands before the CTA exits, including a tile whose list came out empty (no MMA
    // waits for it); for the others the phase has completed already.
    if (lane == 0)
      for (int t = 0; t < KT; ++t)
        if (qearly[t]) drain_wait(cx.bar(B_Q + t), 0);
  } else if (warp == L::kMmaWarp) {
    // ------------------------------ MMA issuer ----------------------------
    if (lane == 0 && nmax > 0) {
      const uint32_t id_qk = tc::idesc_bf16_f32(128, 128, false);
      const uint32_t id_pv = tc::idesc_bf16_f32(128, 128, true);
      const bool rot = p.rope_cos != nullptr;  // Q_t ready: landed (B_Q + t), or both landed and rotated (B_QR)
      bool ok = true;
      // S_t(0) for both tiles.
#pragma unroll
      for (int t = 0; t < KT; ++t) {
        if (!ok || tl[t].n == 0) continue;
        if (!wait_bar(cx, cx.bar(rot ? B_QR : B_Q + t), 0) || !wait_bar(cx, cx.bar(B_KF + t), 0)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        const uint32_t sQ = cx.sbase + L::off_q(t), sK = cx.sbase + L::off_k(t);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kSub + (kk & 3) * 32;
          tc::mma_bf16_ss(tmem + L::col_s(t), tc::sw128_desc(sQ + off, 16, 1024), tc::sw128_desc(sK + off, 16, 1024),
                          id_qk, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(cx.bar(B_KE + t));
        tc::mma_commit(cx.bar(B_SF + t));
      }
      for (int it = 0; ok && it < nmax; ++it) {
#pragma unroll
        for (int t = 0; t < KT; ++t) {
          if (!ok || it >= tl[t].n) continue;
          // O_t += P_t(it) V_t(it), in two parts: keys [0, 64) as soon as the softmax threads have
          // written them, while they still compute the rest; then keys [64, 128).
          if (!wait_bar(cx, cx.bar(B_PH + t), it & 1) || !wait_bar(cx, cx.bar(B_VF + t), it & 1)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t sV = cx.sbase + L::off_v(t);
          // P keys [16 kk, 16 kk + 16) as bf16 pairs in S columns [8 kk, 8 kk + 8)
          auto pv = [&](int kk, uint32_t acc) {
            tc::mma_bf16_ts(tmem + L::col_o(t), tmem + L::col_s(t) + kk * 8,
                            tc::sw128_desc(sV + kk * 2048, kSub, 1024), id_pv, acc);
          };
          pv(0, it > 0 ? 1u : 0u);
          pv(1, 1u);
          pv(2, 1u);
          pv(3, 1u);
          if (!wait_bar(cx, cx.bar(B_PF + t), it & 1)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          pv(4, 1u);
          pv(5, 1u);
          pv(6, 1u);
          pv(7, 1u);
          tc::mma_commit(cx.bar(B_VE + t));
          if (it + 1 < tl[t].n) {
            // S_t(it + 1) = Q_t K_t(it + 1)^T overwrites the TMEM columns holding P_t(it): issue it
            // only once the P.V above has completed (MMAs into different accumulators are not
            // ordered against each other).
            if (!wait_bar(cx, cx.bar(B_VE + t), it & 1)) { ok = false; break; }
            if (!wait_bar(cx, cx.bar(B_KF + t), (it + 1) & 1)) { ok = false; break; }
            tc::tc_fence_after();
            const uint32_t sQ = cx.sbase + L::off_q(t), sK = cx.sbase + L::off_k(t);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t off = (kk >> 2) * kSub + (kk & 3) * 32;
              tc::mma_bf16_ss(tmem + L::col_s(t), tc::sw128_desc(sQ + off, 16, 1024),
                              tc::sw128_desc(sK + off, 16, 1024), id_qk, kk > 0 ? 1u : 0u);
            }
            tc::mma_commit(cx.bar(B_KE + t));
            tc::mma_commit(cx.bar(B_SF + t));
          } else {
            tc::mma_commit(cx.bar(B_OD + t));
          }
        }
      }
      // All MMAs issued by this thread complete before teardown.
      tc::mma_commit(cx.bar(B_DRAIN));
      drain_wait(cx.bar(B_DRAIN), 0);
    }
  } else {
    // ------------------------------ softmax -------------------------------
    const int t = warp >> 2;                 // tile of this warp
    const int r = ((warp & 3) << 5) | lane;  // query row = TMEM lane
    const Tile x = t == 0 ? tl[0] : tl[1];
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + L::col_s(t);  // row r of S_t; P_t in its first 64 columns
    const uint32_t tO = tmem + lane_base + L::col_o(t);  // row r of O_t
    const int qt = x.i * 128 + r;
    const float sl2 = p.scale * 1.4426950408889634f;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    if (p.rope_cos != nullptr && nmax > 0) {
      // RoPE on load: all softmax threads rotate the CTA's Q tiles, then one arrival each on B_QR.
      ok = rope_q_on_load<KT>(cx.abort_flag, cx.status, cx.bar(B_Q), sm, p.rope_cos, p.rope_sin, tl[0].i, tl[1].i,
                              tl[0].n, tl[1].n, warp * 32 + lane);
      tc::mbar_arrive(cx.bar(B_QR));
    }
    for (int it = 0; ok && it < x.n; ++it) {
      ok = __all_sync(0xffffffffu, wait_bar(cx, cx.bar(B_SF + t), it & 1));
      if (!ok) break;
      tc::tc_fence_after();
      const int j = slist[t * kMaxList + it];
      // keys c (0..127 of the block) with c <= lim are visible
      const int lim = (p.causal && j * 128 + 127 > qt) ? qt - j * 128 : 127;
      // The whole row of S_t in registers: its maximum, then P from the same registers.
      uint32_t sv[4][32];
#pragma unroll
      for (int q = 0; q < 4; ++q) tc::tmem_ld32(tS + 32 * q, sv[q]);
      tc::tmem_wait_ld();
      if (lim < 127) {  // causal diagonal: keys beyond the query row are masked
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (32 * q + e > lim) sv[q][e] = __float_as_uint(-INFINITY);
      }
      float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int e = 0; e < 32; e += 8)
#pragma unroll
          for (int u = 0; u < 4; ++u)
            mq[u] = tc::max3(mq[u], __uint_as_float(sv[q][e + 2 * u]), __uint_as_float(sv[q][e + 2 * u + 1]));
      const float mx = tc::max3(mq[0], mq[1], fmaxf(mq[2], mq[3]));
      const float mnew = fmaxf(m, mx * sl2);
      const bool need = mnew > m + kRescaleThreshold || (m == -INFINITY && mnew != -INFINITY);
      // O_t is stable here: PV_t(it-1) completed before S_t(it) was signalled.
      if (__any_sync(0xffffffffu, need) && it > 0) {
        const float f = need ? exp2f(m - mnew) : 1.f;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {  // 16 columns at a time: the row of S_t is live in registers
          uint32_t v[16];
          tc::tmem_ld16(tO + c * 16, v);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * f);
          tc::tmem_st16(tO + c * 16, v);
        }
      }
      if (need) {
        l *= exp2f(m - mnew);
        m = mnew;
      }
      const float nmu = (m == -INFINITY) ? 0.f : -m;
      // P = 2^(s * scale * log2e - m) as bf16 pairs, 16 keys at a time: keys [16 c, 16 c + 16) into
      // S columns [8 c, 8 c + 8) (the whole row is already in registers).  Keys [0, 64) are
      // signalled on their own (B_PH) so that the tensor core starts on them.
      const uint64_t sl2x2 = tc::f2_pack(sl2, sl2), nmux2 = tc::f2_pack(nmu, nmu);
      uint64_t acc[4] = {0, 0, 0, 0};  // packed (even, odd) column partial row sums
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t* cur = &sv[c >> 1][(c & 1) * 16];
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          float a0, a1;
          tc::f2_unpack(tc::f2_fma(tc::f2_pack(__uint_as_float(cur[e]), __uint_as_float(cur[e + 1])), sl2x2,
                                   nmux2), a0, a1);
          const float p0 = tc::ex2_approx(a0), p1 = tc::ex2_approx(a1);
          acc[(e >> 1) & 3] = tc::f2_add(acc[(e >> 1) & 3], tc::f2_pack(p0, p1));
          pk[e >> 1] = pack_bf16x2(p0, p1);
        }
        tc::tmem_st8(tS + c * 8, pk);
        if (c == 3) {  // keys [0, 64) written: the tensor core may start on them
          tc::tmem_wait_st();
          tc::tc_fence_before();
          tc::mbar_arrive(cx.bar(B_PH + t));
        }
      }
      float rs0, rs1, rs2, rs3;
      tc::f2_unpack(tc::f2_add(acc[0], acc[1]), rs0, rs1);
      tc::f2_unpack(tc::f2_add(acc[2], acc[3]), rs2, rs3);
      l += (rs0 + rs1) + (rs2 + rs3);
      tc::tmem_wait_st();
      tc::tc_fence_before();
      tc::mbar_arrive(cx.bar(B_PF + t));
    }
    if (x.n > 0 && ok) ok = __all_sync(0xffffffffu, wait_bar(cx, cx.bar(B_OD + t), 0));
    // ok and x.n are uniform over the tile's warps.
    if (x.valid && (x.n == 0 || ok)) {
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.O) + ((size_t)(x.b * p.Hq + x.h) * p.L + qt) * kHD;
      if (x.n > 0) {
        tc::tc_fence_after();
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tc::tmem_ld32(tO + c * 32, v);
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
      } else {
#pragma unroll
        for (int q = 0; q < 16; ++q) reinterpret_cast<uint4*>(orow)[q] = make_uint4(0, 0, 0, 0);
      }
      if (p.lse != nullptr)
        p.lse[(size_t)(x.b * p.Hq + x.h) * p.L + qt] =
            (x.n > 0 && l > 0.f) ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == L::kMmaWarp) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

template <int KT>
static cudaError_t launch_attn_t(const AttnParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                 const CUtensorMap& tmV, cudaStream_t st) {
  using L = Layout<KT>;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<KT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)L::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  if (KT == 1) {  // room for two CTAs per SM
    e = cudaFuncSetAttribute(attn_tc_kernel<KT>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
  }
  const size_t tiles = (size_t)p.B * p.Hq * p.nb;
  const unsigned grid = (unsigned)((tiles + KT - 1) / KT);
  attn_tc_kernel<KT><<<grid, L::kThreads, L::SMEM_BYTES, st>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

// Short index lists (few key blocks per query tile) leave each CTA's prologue and epilogue
// exposed: one tile per CTA lets two CTAs per SM hide them behind each other.  Long lists
// favour the two-tile ping-pong inside one CTA.  (Measured on this B200, one vs two tiles per
// CTA: 64K layer at 1% density (lists of 3) 0.78 vs 0.85 ms; at 25% (69) 9.2 vs 9.0 ms; the
// 32K layer (14) 1.077 vs 1.066 ms; the 128K layer (26) within run-to-run noise.)
constexpr int kShortList = 12;

cudaError_t launch_attn_tcgen05(const AttnParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                const CUtensorMap& tmV, cudaStream_t st) {
  return p.kmax <= kShortList ? launch_attn_t<1>(p, tmQ, tmK, tmV, st) : launch_attn_t<2>(p, tmQ, tmK, tmV, st);
}

}  // namespace sfa
