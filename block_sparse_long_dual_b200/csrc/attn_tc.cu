// Exact attention over the kept key blocks ("Prism: Spectral-Aware
// Block-Sparse Attention" §1) on the sm_100a tensor cores.
//
// bf16 Q/K/V, query block = key block = 128 tokens, head dim 128.
// Persistent: one CTA per SM, resident for the whole launch.  A CTA runs two
// independent query-tile streams ("slots"); slot t of CTA c takes the tiles
// 2 c + t, 2 c + t + 2 G, ... (G = grid size) of the order (b, kv head, query
// block descending, q head in the group), so the longest lists go first.  The
// two slots ping-pong on the tensor core: while one slot's softmax turns S
// into P, the tensor core runs the other slot's P.V and next Q.K^T.  Because
// the CTA stays resident, a slot's next tile (its index list, Q tile and
// first K tile, and its first Q.K^T) is prepared while that slot is still
// finishing the previous tile's last block and epilogue.
//
//   warps 0 .. 15    softmax of slot w / 8: two threads per query row r (TMEM
//                    lane r; warps w and w+4 share lanes), each owning 64 of the
//                    128 key columns, row maxima exchanged through shared
//                    memory; reads S from TMEM, online softmax with a lazily
//                    rescaled O, writes P (bf16) back into the S columns of
//                    TMEM, final O / l epilogue straight from TMEM to global.
//   warp 16          producer: validates each tile's index list into shared
//                    memory, then TMA loads of Q and of K(j), V(j) for every
//                    kept block j (one K and one V slot per query slot).
//   warp 17          MMA issuer: S = Q K^T (A, B from shared memory) and
//                    O += P V (A = P from TMEM, B = V from shared memory),
//                    M = N = 128, K = 16 steps; completion tracked with
//                    tcgen05.commit -> mbarriers.  A commit covers every MMA the
//                    thread issued before it, so the commit that signals S(j)
//                    also means O has absorbed P(j-1).
// TMEM (512 columns): S_t at [128 t, 128 t + 128), O_t at [256 + 128 t, +128);
// P_t aliases S_t (two bf16 per column): keys [0,64) in S columns [0,32), keys
// [64,128) in S columns [64,96), each half written by the threads that read it.
//
// Flow control per slot: index lists in a ring of two shared-memory buffers
// (full / empty barriers); Q, K and V slots reused once the MMAs that read them
// have completed; O reused once the epilogue has read it.  Every mbarrier wait
// is bounded (about 2 s); a wait that runs out writes SFA_ERR_TIMEOUT to the
// status word, raises a CTA-wide abort flag, drains the copies / MMAs this CTA
// issued and frees its tensor memory.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace sfa {

namespace {

constexpr int kHD = 128;
constexpr uint32_t kSub = 16384;       // 128 rows x 64 bf16 (one 128B-swizzle box)
constexpr uint32_t kTile = 2 * kSub;   // 128 x 128 bf16
constexpr int kMaxList = 2048;         // nb <= 2048, so a valid list has <= 2048 entries
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8

// Barriers, one per slot unless noted.
enum {
  B_Q = 0,        // Q tile landed (TMA)
  B_KF = 2,       // K tile landed
  B_VF = 4,       // V tile landed
  B_KE = 6,       // K slot free (the Q.K^T that read it completed)
  B_VE = 8,       // V slot free (the P.V that read it completed)
  B_SF = 10,      // S in TMEM
  B_PF = 12,      // P in TMEM (256 softmax arrivals)
  B_OD = 14,      // every P.V of the tile completed
  B_OFREE = 16,   // the epilogue has read O (256 arrivals)
  B_QR = 18,      // Q rotated in shared memory (RoPE on load; 256 arrivals)
  B_LFULL = 20,   // [slot][buffer] index list validated (32 producer arrivals)
  B_LEMPTY = 24,  // [slot][buffer] index list consumed (256 softmax + 1 MMA arrivals)
  B_X = 28,       // [slot][warp pair][parity] row-max / row-sum exchange of warps w and w + 4 (64 arrivals)
  B_DRAIN = 44,
  NBAR = 45
};

// Shared memory: per slot a Q, a K and a V tile, then barriers, counts, exchange, lists.
__host__ __device__ constexpr uint32_t off_q(int t) { return t * kTile; }
__host__ __device__ constexpr uint32_t off_k(int t) { return (2 + t) * kTile; }
__host__ __device__ constexpr uint32_t off_v(int t) { return (4 + t) * kTile; }
constexpr uint32_t OFF_BAR = 6 * kTile;
constexpr uint32_t OFF_MISC = OFF_BAR + ((NBAR * 8 + 15) & ~15);  // tmem slot, abort flag, counts [slot][buffer]
constexpr uint32_t OFF_XCHG = OFF_MISC + 32;                      // [slot][parity][half][row] float
constexpr uint32_t OFF_LIST = OFF_XCHG + 2 * 2 * 2 * 128 * 4;     // [slot][buffer][kMaxList] uint16
constexpr uint32_t SMEM_BYTES = OFF_LIST + 2 * 2 * kMaxList * 2 + 1024;
constexpr int kThreads = 2 * 256 + 64;
constexpr int kProducerWarp = 16, kMmaWarp = 17;
constexpr uint32_t TMEM_COLS = 512;
__host__ __device__ constexpr uint32_t col_s(int t) { return t * 128; }
__host__ __device__ constexpr uint32_t col_o(int t) { return 256 + t * 128; }
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");

struct Ctx {
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
  int b, h, g, i;
  bool valid;
};

// Tile q of the order (b, kv head, query block descending, q head in the group).
__device__ Tile decode_tile(const AttnParams& p, int q) {
  Tile x;
  const int group = p.Hq / p.Hkv;
  const int total = p.B * p.Hq * p.nb;
  x.valid = q < total;
  if (!x.valid) q = total - 1;
  const int hh = q % group;
  q /= group;
  x.i = p.nb - 1 - (q % p.nb);
  q /= p.nb;
  x.g = q % p.Hkv;
  x.b = q / p.Hkv;
  x.h = x.g * group + hh;
  return x;
}

// The r-th tile of slot t of this CTA.
__device__ __forceinline__ int slot_tile(int r, int t) { return (r * (int)gridDim.x + (int)blockIdx.x) * 2 + t; }

// RoPE on load: the slot's 256 softmax threads rotate its Q tile in shared memory once the TMA
// copy has landed (bounded wait on B_Q); returns false if the wait gave up.  Work unit = (row,
// 16-byte chunk c): chunk c of box 0 holds dims [8c, 8c + 8) and the same offset of box 1 holds
// their rotary partners [64 + 8c, 64 + 8c + 8) (chunk c of row r is stored at chunk c ^ (r & 7)
// of the 128-byte row).  Thread st takes chunk st & 7 of rows st / 8 + 32 k (k < 4), so a warp
// touches four whole rows: conflict-free in shared memory, and each row's table entries are one
// contiguous 256-byte run.  The table entries are fetched before the wait, so their latency
// hides behind the copy.  Kept out of line: it runs once per tile and must not add to the
// register pressure of the softmax loop.
__device__ __noinline__ bool rope_q_on_load(volatile int* abort_flag, int* status, uint32_t bar_q, uint32_t parity,
                                            unsigned char* sq, const float* cos_t, const float* sin_t, int i, int st) {
  Ctx cx;
  cx.bars = 0;
  cx.abort_flag = abort_flag;
  cx.status = status;
  const int c = st & 7;
  float ca[4][8], sa[4][8];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int row = (st >> 3) + 32 * k;
    load8(cos_t + ((size_t)i * 128 + row) * 64 + c * 8, ca[k]);
    load8(sin_t + ((size_t)i * 128 + row) * 64 + c * 8, sa[k]);
  }
  if (!__all_sync(0xffffffffu, wait_bar(cx, bar_q, parity))) return false;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int row = (st >> 3) + 32 * k;
    unsigned char* rp = sq + row * 128 + ((c ^ (row & 7)) << 4);
    uint4* plo = reinterpret_cast<uint4*>(rp);
    uint4* phi = reinterpret_cast<uint4*>(rp + kSub);
    const uint4 ulo = *plo, uhi = *phi;
    const uint32_t wl[4] = {ulo.x, ulo.y, ulo.z, ulo.w}, wh[4] = {uhi.x, uhi.y, uhi.z, uhi.w};
    uint32_t ol[4], oh[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float l0, l1, h0, h1;
      rope_pair(__uint_as_float(wl[e] << 16), __uint_as_float(wh[e] << 16), ca[k][2 * e], sa[k][2 * e], l0, h0);
      rope_pair(__uint_as_float(wl[e] & 0xFFFF0000u), __uint_as_float(wh[e] & 0xFFFF0000u), ca[k][2 * e + 1],
                sa[k][2 * e + 1], l1, h1);
      ol[e] = pack_bf16x2(l0, l1);
      oh[e] = pack_bf16x2(h0, h1);
    }
    *plo = make_uint4(ol[0], ol[1], ol[2], ol[3]);
    *phi = make_uint4(oh[0], oh[1], oh[2], oh[3]);
  }
  tc::fence_proxy_async_smem();  // the generic-proxy writes become visible to the MMAs
  return true;
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, AttnParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  unsigned char* sm = smem_raw + pad;
  const uint32_t sbase = raw + pad;
  Ctx cx;
  cx.bars = sbase + OFF_BAR;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  cx.abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);
  volatile int* nsh = reinterpret_cast<volatile int*>(sm + OFF_MISC + 8);    // [slot][buffer] list counts
  uint16_t* slist = reinterpret_cast<uint16_t*>(sm + OFF_LIST);              // [slot][buffer][kMaxList]
  cx.status = p.status;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    *cx.abort_flag = 0;
    for (int k = 0; k < NBAR; ++k) {
      uint32_t cnt = 1;
      if (k == B_PF || k == B_PF + 1 || k == B_OFREE || k == B_OFREE + 1 || k == B_QR || k == B_QR + 1)
        cnt = 256;
      else if (k >= B_LFULL && k < B_LFULL + 4)
        cnt = 32;
      else if (k >= B_LEMPTY && k < B_LEMPTY + 4)
        cnt = 257;
      else if (k >= B_X && k < B_X + 16)
        cnt = 64;
      tc::mbar_init(cx.bar(k), cnt);
    }
    tc::fence_mbar_init();
  } else if (warp == kProducerWarp && lane == 0) {
    tc::prefetch_tmap(&tmQ);
    tc::prefetch_tmap(&tmK);
    tc::prefetch_tmap(&tmV);
  } else if (warp == kMmaWarp) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool rot = p.rope_cos != nullptr;  // Q ready: landed (B_Q), or landed and rotated (B_QR)

  if (warp == kProducerWarp) {
    // ------------------------------ producer ------------------------------
    // A polling state machine per slot (never blocks on one slot while the other could move):
    // LIST (validate the next tile's list once its ring buffer is free), K (load K(it), and Q
    // first, once the slot's last Q.K^T completed), V (load V(it) once the last P.V completed).
    enum { P_LIST, P_K, P_V, P_DONE };
    int state[2] = {P_LIST, P_LIST}, r[2] = {0, 0}, it[2] = {0, 0}, n[2] = {0, 0};
    int nk[2] = {0, 0}, nv[2] = {0, 0}, nq[2] = {0, 0};  // loads issued
    Tile xs[2] = {decode_tile(p, slot_tile(0, 0)), decode_tile(p, slot_tile(0, 1))};  // each slot's current tile
    uint64_t last = globaltimer_ns();
    bool ok = true;
    for (uint32_t spin = 0; ok && !(state[0] == P_DONE && state[1] == P_DONE); ++spin) {
      bool moved = false;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const Tile x = xs[t];
        const int buf = r[t] & 1;
        if (state[t] == P_LIST) {
          if (!x.valid) {
            state[t] = P_DONE;
            continue;
          }
          bool ready = r[t] < 2 || tc::mbar_test_wait(cx.bar(B_LEMPTY + 2 * t + buf), ((r[t] >> 1) - 1) & 1);
          if (!__shfl_sync(0xffffffffu, ready, 0)) continue;
          // Validate the list: count in [0, kmax], entries ascending in [0, nb), <= i if causal.
          const size_t rowid = (size_t)(x.b * p.Hq + x.h) * p.nb + x.i;
          const int* src = p.idx + rowid * p.kmax;
          int cnt = p.counts[rowid];
          bool good = cnt >= 0 && cnt <= p.kmax;
          if (good) {
            for (int u = lane; u < cnt; u += 32) {
              const int j = src[u];
              if (j < 0 || j >= p.nb || (p.causal && j > x.i) || (u > 0 && src[u - 1] >= j)) good = false;
              if (u < kMaxList) slist[(t * 2 + buf) * kMaxList + u] = (uint16_t)j;
            }
          }
          good = __all_sync(0xffffffffu, good);
          if (!good) {
            if (lane == 0) report(p.status, SFA_ERR_INDEX);
            cnt = 0;
          }
          if (lane == 0) nsh[t * 2 + buf] = cnt;
          __syncwarp();
          tc::mbar_arrive(cx.bar(B_LFULL + 2 * t + buf));
          moved = true;
          if (cnt == 0) {
            xs[t] = decode_tile(p, slot_tile(++r[t], t));
          } else {
            n[t] = cnt;
            it[t] = 0;
            state[t] = P_K;
          }
        } else if (state[t] == P_K) {
          // K slot (and, at a tile's first block, the Q slot) free once the slot's last Q.K^T completed
          bool ready = nk[t] == 0 || tc::mbar_test_wait(cx.bar(B_KE + t), (nk[t] - 1) & 1);
          if (!__shfl_sync(0xffffffffu, ready, 0)) continue;
          if (lane == 0) {
            if (it[t] == 0) {
              const int qrow = (x.b * p.Hq + x.h) * p.L + x.i * 128;
              const uint32_t sQ = sbase + off_q(t);
              tc::mbar_arrive_expect_tx(cx.bar(B_Q + t), kTile);
              tc::tma_load_2d(sQ, &tmQ, cx.bar(B_Q + t), 0, qrow);
              tc::tma_load_2d(sQ + kSub, &tmQ, cx.bar(B_Q + t), 64, qrow);
            }
            const int row = (x.b * p.Hkv + x.g) * p.L + (int)slist[(t * 2 + buf) * kMaxList + it[t]] * 128;
            const uint32_t sK = sbase + off_k(t);
            tc::mbar_arrive_expect_tx(cx.bar(B_KF + t), kTile);
            tc::tma_load_2d(sK, &tmK, cx.bar(B_KF + t), 0, row);
            tc::tma_load_2d(sK + kSub, &tmK, cx.bar(B_KF + t), 64, row);
          }
          if (it[t] == 0) ++nq[t];
          ++nk[t];
          state[t] = P_V;
          moved = true;
        } else if (state[t] == P_V) {
          bool ready = nv[t] == 0 || tc::mbar_test_wait(cx.bar(B_VE + t), (nv[t] - 1) & 1);
          if (!__shfl_sync(0xffffffffu, ready, 0)) continue;
          if (lane == 0) {
            const int row = (x.b * p.Hkv + x.g) * p.L + (int)slist[(t * 2 + buf) * kMaxList + it[t]] * 128;
            const uint32_t sV = sbase + off_v(t);
            tc::mbar_arrive_expect_tx(cx.bar(B_VF + t), kTile);
            tc::tma_load_2d(sV, &tmV, cx.bar(B_VF + t), 0, row);
            tc::tma_load_2d(sV + kSub, &tmV, cx.bar(B_VF + t), 64, row);
          }
          ++nv[t];
          moved = true;
          if (++it[t] == n[t]) {
            xs[t] = decode_tile(p, slot_tile(++r[t], t));
            state[t] = P_LIST;
          } else {
            state[t] = P_K;
          }
        }
      }
      if (moved) {
        last = globaltimer_ns();
      } else {
        __nanosleep(64);  // nothing ready: leave the issue slots to the softmax warps for a moment
      }
      if (!moved && (spin & 15u) == 0) {
        bool stop = *cx.abort_flag != 0;
        if (!stop && globaltimer_ns() - last > kTimeoutNs) {
          if (lane == 0) {
            *cx.abort_flag = 1;
            report(cx.status, SFA_ERR_TIMEOUT);
          }
          stop = true;
        }
        ok = !__shfl_sync(0xffffffffu, stop, 0);
      }
    }
    __syncwarp();
    if (*cx.abort_flag && lane == 0) {
      // Let every copy this CTA started land before the CTA exits.
      for (int t = 0; t < 2; ++t) {
        if (nq[t] > 0) drain_wait(cx.bar(B_Q + t), (nq[t] - 1) & 1);
        if (nk[t] > 0) drain_wait(cx.bar(B_KF + t), (nk[t] - 1) & 1);
        if (nv[t] > 0) drain_wait(cx.bar(B_VF + t), (nv[t] - 1) & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------ MMA issuer ----------------------------
    // A polling state machine per slot: NEW (read the next tile's list count), S0 (the tile's
    // first Q.K^T), PV (O += P V), S (the next Q.K^T).  Whichever slot is ready goes next, so the
    // two slots' MMAs interleave as their softmax results arrive.
    if (lane == 0) {
      enum { M_NEW, M_S0, M_PV, M_S, M_DONE };
      const uint32_t id_qk = tc::idesc_bf16_f32(128, 128, false);
      const uint32_t id_pv = tc::idesc_bf16_f32(128, 128, true);
      int state[2] = {M_NEW, M_NEW}, r[2] = {0, 0}, it[2] = {0, 0}, n[2] = {0, 0}, ne[2] = {0, 0};
      int ns[2] = {0, 0}, npv[2] = {0, 0};  // Q.K^T and P.V issued
      uint64_t last = globaltimer_ns();
      int idle = 0;
      auto ready = [&](int k, uint32_t parity) { return tc::mbar_test_wait(cx.bar(k), parity); };
      auto issue_s = [&](int t) {
        tc::tc_fence_after();
        const uint32_t sQ = sbase + off_q(t), sK = sbase + off_k(t);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kSub + (kk & 3) * 32;
          tc::mma_bf16_ss(tmem + col_s(t), tc::sw128_desc(sQ + off, 16, 1024), tc::sw128_desc(sK + off, 16, 1024),
                          id_qk, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(cx.bar(B_KE + t));
        tc::mma_commit(cx.bar(B_SF + t));
        ++ns[t];
      };
      for (uint32_t spin = 0; !(state[0] == M_DONE && state[1] == M_DONE); ++spin) {
        bool moved = false;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (state[t] == M_NEW) {
            if (slot_tile(r[t], t) >= p.B * p.Hq * p.nb) {
              state[t] = M_DONE;
              continue;
            }
            const int buf = r[t] & 1;
            if (!ready(B_LFULL + 2 * t + buf, (r[t] >> 1) & 1)) continue;
            n[t] = nsh[t * 2 + buf];
            tc::mbar_arrive(cx.bar(B_LEMPTY + 2 * t + buf));
            ++r[t];
            moved = true;
            if (n[t] > 0) state[t] = M_S0;
          } else if (state[t] == M_S0) {
            // S(0) overwrites the P columns the slot's last P.V read: that P.V must have completed.
            if ((npv[t] > 0 && !ready(B_VE + t, (npv[t] - 1) & 1)) || !ready(rot ? B_QR + t : B_Q + t, ne[t] & 1) ||
                !ready(B_KF + t, ns[t] & 1))
              continue;
            issue_s(t);
            it[t] = 0;
            state[t] = M_PV;
            moved = true;
          } else if (state[t] == M_PV) {
            // The first P.V of a tile overwrites O: the previous tile's epilogue must have read it.
            if (!ready(B_PF + t, npv[t] & 1) || !ready(B_VF + t, npv[t] & 1) ||
                (it[t] == 0 && ne[t] > 0 && !ready(B_OFREE + t, (ne[t] - 1) & 1)))
              continue;
            tc::tc_fence_after();
            const uint32_t sV = sbase + off_v(t);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              // P keys [16 kk, 16 kk + 16): half kk / 4 wrote them into its own S columns
              tc::mma_bf16_ts(tmem + col_o(t), tmem + col_s(t) + (kk >> 2) * 64 + (kk & 3) * 8,
                              tc::sw128_desc(sV + kk * 2048, kSub, 1024), id_pv, (it[t] > 0 || kk > 0) ? 1u : 0u);
            tc::mma_commit(cx.bar(B_VE + t));
            ++npv[t];
            if (++it[t] < n[t]) {
              state[t] = M_S;
            } else {
              tc::mma_commit(cx.bar(B_OD + t));
              ++ne[t];
              state[t] = M_NEW;
            }
            moved = true;
          } else if (state[t] == M_S) {
            // S(it) overwrites the TMEM columns holding P(it - 1): issue it only once the P.V that
            // read them has completed (MMAs into different accumulators are not ordered).
            if (!ready(B_VE + t, (npv[t] - 1) & 1) || !ready(B_KF + t, ns[t] & 1)) continue;
            issue_s(t);
            state[t] = M_PV;
            moved = true;
          }
        }
        if (moved) {
          last = globaltimer_ns();
          continue;
        }
        // Nothing ready: let the hardware suspend this thread on one slot's next barrier (it
        // resumes as soon as that phase completes, or after ~0.5 us to look at the other slot), so
        // the issue slots it shares with the softmax warps are not spent polling.
        idle ^= 1;
        int kb = -1;
        uint32_t kp = 0;
#pragma unroll
        for (int t = 0; t < 2; ++t) {  // static indices only: the per-slot state stays in registers
          const bool pick = (t == idle && state[t] != M_DONE) || (t != idle && state[1 - t] == M_DONE);
          if (!pick || kb >= 0) continue;
          if (state[t] == M_NEW) { kb = B_LFULL + 2 * t + (r[t] & 1); kp = (r[t] >> 1) & 1; }
          else if (state[t] == M_S0) { kb = B_KF + t; kp = ns[t] & 1; }
          else if (state[t] == M_PV) { kb = B_PF + t; kp = npv[t] & 1; }
          else if (state[t] == M_S) { kb = B_VE + t; kp = (npv[t] - 1) & 1; }
        }
        if (kb >= 0) tc::mbar_try_wait_ns(cx.bar(kb), kp, 500);
        if ((spin & 15u) == 0) {
          if (*cx.abort_flag) break;
          if (globaltimer_ns() - last > kTimeoutNs) {
            *cx.abort_flag = 1;
            report(cx.status, SFA_ERR_TIMEOUT);
            break;
          }
        }
      }
      // All MMAs issued by this thread complete before teardown.
      tc::mma_commit(cx.bar(B_DRAIN));
      drain_wait(cx.bar(B_DRAIN), 0);
    }
  } else {
    // ------------------------------ softmax -------------------------------
    const int t = warp >> 3;                 // slot of this warp
    const int hf = (warp >> 2) & 1;          // key-column half: [64 hf, 64 hf + 64)
    const int rr = ((warp & 3) << 5) | lane;  // query row = TMEM lane
    const int st = (warp & 7) * 32 + lane;   // thread index within the slot
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + col_s(t) + 64 * hf;     // this half's S columns
    const uint32_t tP = tS;                                         // this half's P columns (2 bf16 each)
    const uint32_t tO = tmem + lane_base + col_o(t) + 64 * hf;     // this half's O columns
    // Exchange with the other thread of the row (same lane, warp w ^ 4, on the same SM
    // sub-partition): write this half's value, arrive on the pair's barrier of parity u & 1 (64
    // arrivals), wait (the hardware suspends the warp meanwhile), read the partner's value.  Use u
    // waits for phase (u / 2) & 1 of its barrier; the buffer of parity u & 1 is rewritten by use
    // u + 2 only after both threads passed use u + 1.
    float* xchg = reinterpret_cast<float*>(sm + OFF_XCHG) + t * 512;  // [parity][half][row]
    const uint32_t xbar = cx.bar(B_X + t * 8 + (warp & 3) * 2);
    uint32_t xuse = 0;
    auto exchange = [&](float v) -> float {
      const uint32_t use = xuse++;
      float* xc = xchg + (use & 1) * 256;
      xc[hf * 128 + rr] = v;
      const uint32_t xb = xbar + 8u * (use & 1);
      tc::mbar_arrive(xb);
      if (!wait_bar(cx, xb, (use >> 1) & 1)) return NAN;
      return xc[(1 - hf) * 128 + rr];
    };
    const float sl2 = p.scale * 1.4426950408889634f;
    int blk = 0, ne = 0;  // blocks and non-empty tiles processed
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const Tile x = decode_tile(p, slot_tile(r, t));
      if (!x.valid) break;
      const int buf = r & 1;
      ok = __all_sync(0xffffffffu, wait_bar(cx, cx.bar(B_LFULL + 2 * t + buf), (r >> 1) & 1));
      if (!ok) break;
      const int n = nsh[t * 2 + buf];
      const uint32_t lst = (uint32_t)(t * 2 + buf) * kMaxList;  // this tile's list in slist
      const int qt = x.i * 128 + rr;
      if (n == 0) {
        __nv_bfloat16* orow =
            static_cast<__nv_bfloat16*>(p.O) + ((size_t)(x.b * p.Hq + x.h) * p.L + qt) * kHD + 64 * hf;
        tc::mbar_arrive(cx.bar(B_LEMPTY + 2 * t + buf));
#pragma unroll
        for (int q = 0; q < 8; ++q) reinterpret_cast<uint4*>(orow)[q] = make_uint4(0, 0, 0, 0);
        if (p.lse != nullptr && hf == 0) p.lse[(size_t)(x.b * p.Hq + x.h) * p.L + qt] = -INFINITY;
        continue;
      }
      if (rot) {
        // RoPE on load: the slot's 256 threads rotate its Q tile, then one arrival each on B_QR.
        ok = rope_q_on_load(cx.abort_flag, cx.status, cx.bar(B_Q + t), ne & 1, sm + off_q(t), p.rope_cos,
                            p.rope_sin, x.i, st);
        tc::mbar_arrive(cx.bar(B_QR + t));
        if (!ok) break;
      }
      float m = -INFINITY, l = 0.f;  // l: this half's share of the row sum
      for (int it = 0; ok && it < n; ++it, ++blk) {
        ok = __all_sync(0xffffffffu, wait_bar(cx, cx.bar(B_SF + t), blk & 1));
        if (!ok) break;
        tc::tc_fence_after();
        const int j = slist[lst + it];
        // keys c (0..127 of the block) with c <= lim are visible; this half holds c = 64 hf + cc
        const int lim = ((p.causal && j * 128 + 127 > qt) ? qt - j * 128 : 127) - 64 * hf;
        // Pass 1: max over this half, then the row max through shared memory.
        float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        {
          uint32_t sv[2][32];
          tc::tmem_ld32(tS, sv[0]);
          tc::tmem_ld32(tS + 32, sv[1]);
          tc::tmem_wait_ld();
          if (lim < 63) {  // causal diagonal: keys beyond the query row are masked
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (c * 32 + e > lim) sv[c][e] = __float_as_uint(-INFINITY);
          }
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int e = 0; e < 32; e += 8)
#pragma unroll
              for (int q = 0; q < 4; ++q)
                mq[q] = tc::max3(mq[q], __uint_as_float(sv[c][e + 2 * q]), __uint_as_float(sv[c][e + 2 * q + 1]));
        }
        const float mhalf = tc::max3(mq[0], mq[1], fmaxf(mq[2], mq[3]));
        const float mx = fmaxf(mhalf, exchange(mhalf));
        const float mnew = fmaxf(m, mx * sl2);
        const bool need = mnew > m + kRescaleThreshold || (m == -INFINITY && mnew != -INFINITY);
        // O is stable here: P.V(it-1) completed before S(it) was signalled.
        if (__any_sync(0xffffffffu, need) && it > 0) {
          const float f = need ? exp2f(m - mnew) : 1.f;
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            uint32_t v[32];
            tc::tmem_ld32(tO + c * 32, v);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * f);
            tc::tmem_st32(tO + c * 32, v);
          }
        }
        if (need) {
          l *= exp2f(m - mnew);
          m = mnew;
        }
        const float nmu = (m == -INFINITY) ? 0.f : -m;
        // Pass 2: P = 2^(s * scale * log2e - m) as bf16 pairs, 16 columns at a time
        // (double-buffered TMEM loads).  P chunk c of this half lands in S columns
        // [64 hf + 8 c, +8), which this thread has already read.
        const uint64_t sl2x2 = tc::f2_pack(sl2, sl2), nmux2 = tc::f2_pack(nmu, nmu);
        uint64_t acc[4] = {0, 0, 0, 0};  // packed (even, odd) column partial row sums
        uint32_t buf2[2][16];
        tc::tmem_ld16(tS, buf2[0]);
        tc::tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t (&cur)[16] = buf2[c & 1];
          if (c < 3) tc::tmem_ld16(tS + (c + 1) * 16, buf2[(c + 1) & 1]);
          if (lim < 63) {
#pragma unroll
            for (int e = 0; e < 16; ++e)
              if (c * 16 + e > lim) cur[e] = __float_as_uint(-INFINITY);
          }
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
          tc::tmem_st8(tP + c * 8, pk);
          if (c < 3) tc::tmem_wait_ld();
        }
        float rs0, rs1, rs2, rs3;
        tc::f2_unpack(tc::f2_add(acc[0], acc[1]), rs0, rs1);
        tc::f2_unpack(tc::f2_add(acc[2], acc[3]), rs2, rs3);
        l += (rs0 + rs1) + (rs2 + rs3);
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tc::mbar_arrive(cx.bar(B_PF + t));
      }
      if (!ok) break;
      tc::mbar_arrive(cx.bar(B_LEMPTY + 2 * t + buf));
      ok = __all_sync(0xffffffffu, wait_bar(cx, cx.bar(B_OD + t), ne & 1));
      if (!ok) break;
      // Epilogue: O / l straight from TMEM to global memory; then O may be overwritten.
      const float ltot = l + exchange(l);
      const Tile y = decode_tile(p, slot_tile(r, t));
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.O) + ((size_t)(y.b * p.Hq + y.h) * p.L + qt) * kHD + 64 * hf;
      tc::tc_fence_after();
      const float inv = ltot > 0.f ? 1.f / ltot : 0.f;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
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
      tc::tc_fence_before();
      tc::mbar_arrive(cx.bar(B_OFREE + t));
      if (p.lse != nullptr && hf == 0)
        p.lse[(size_t)(y.b * p.Hq + y.h) * p.L + qt] = ltot > 0.f ? (m + log2f(ltot)) * 0.6931471805599453f : -INFINITY;
      ++ne;
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

cudaError_t launch_attn_tcgen05(const AttnParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                const CUtensorMap& tmV, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const long long tiles = (long long)p.B * p.Hq * p.nb;
  const long long pairs = (tiles + 1) / 2;
  const unsigned grid = (unsigned)(pairs < sms ? pairs : sms);
  attn_tc_kernel<<<grid, kThreads, SMEM_BYTES, st>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

}  // namespace sfa
