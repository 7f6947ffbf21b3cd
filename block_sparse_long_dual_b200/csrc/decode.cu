// Decode-side estimate -> exact attention ("FASA: Frequency-aware Sparse
// Attention" §2B): one query token per (batch, Q head) against a KV cache.
//
//   fc_gather      compact copy K_fc [B, Hkv, L, 2 nfc] of the dominant rotary
//                  pairs of the rotated key cache (low dims, then partners);
//                  run once over the cache, then per appended token range.
//   tip_chunk      Token Importance Predictor, persistent (one or two CTAs per
//                  SM) over tiles (chunk of C tokens, b, KV head): the chunk's
//                  K_fc rows stream through a bulk-copy ring once for all Q
//                  heads of the group; each token's score is first taken on
//                  the tensor cores in float32 (a filter), then per head a lower bound
//                  of the chunk's k-th largest score (from group maxima),
//                  lowered by twice the float32 chain's rounding bound, and
//                  the tokens at or above it (token order, per warp segment)
//                  get their exact score recomputed in float64.
//   tip_merge      CTA per (b, h): the candidates' float64 keys staged in
//                  shared memory, bounded again, exact k-th largest by radix
//                  select, ties by index; ascending index list, -1 padded (the
//                  same select over global memory when the candidates do not
//                  fit).
//   fac            Focused Attention Computation: CTA per (b, h), 16 warps,
//                  each warp gathers the K / V rows of its share of the kept
//                  tokens (eight tokens' loads in flight per lane), float32
//                  online softmax, warps merged through shared memory.
//
// Ranking: the token score is the dot product over the dominant pairs' dims;
// it is ranked by its float64 value (key = order-preserving uint64 of the
// double, +0 for both zeros); the first k by (key desc, index asc).
//
// Why the float32 filter loses no token of the top k (finite inputs): the
// filter score is a tensor-core sum of n = 2 nfc products, each exact (bf16 x
// bf16); whatever the order and rounding of its float32 accumulation (even
// truncation to 22 bits per addition), it is off the exact score by at most
// n 2^-21 sum_c |q_c k_c| + n 2^-126 (the second term covers flushed
// subnormals), below M = 2^-16 ||q||_1 A + n 2^-126 for n <= 128, where
// sum_c |q_c k_c| <= ||q||_1 A and A = the largest |k| in the chunk's compact
// rows.  If at least k tokens of a chunk have filter scores >= x, they have
// exact scores >= x - M, so the row's k-th largest exact score is >= x - M,
// and every token of the row's top k has a filter score >= x - 2M.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace sfa {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// Order-preserving unsigned keys of float32 (filter) and float64 (ranked) scores.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f == 0.f ? 0.f : f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}
__device__ __forceinline__ uint64_t order_key64(double f) {
  const uint64_t u = (uint64_t)__double_as_longlong(f == 0.0 ? 0.0 : f);
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// The k-th largest of n keys (1 <= k <= n) by MSB-first 8-bit radix select over a
// block of kThreads threads: returns T and sets *gt = #{key > T}.
template <typename Key, typename KeyAt>
__device__ Key block_kth_largest(KeyAt key_at, int n, int k, uint32_t* hist, int* sh, int* gt) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  Key prefix = 0, pmask = 0;
  int krem = k;
  for (int shift = 8 * (int)sizeof(Key) - 8; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kThreads) hist[i] = 0;
    __syncthreads();
    // Warp-aggregated increments: keys cluster in a few digits (float exponents), so lanes with
    // the same digit add once through their lowest lane instead of serialising on one bin.
    for (int i0 = 0; i0 < n; i0 += kThreads) {
      const int i = i0 + tid;
      int bin = -1;
      if (i < n) {
        const Key u = key_at(i);
        if ((u & pmask) == prefix) bin = (int)((u >> shift) & 255u);
      }
      const unsigned same = __match_any_sync(0xffffffffu, bin);
      if (bin >= 0 && lane == __ffs(same) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(same));
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns digits 255 - 8l - j, j = 0..7 (descending)
      uint32_t c[8];
      int s = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = hist[255 - 8 * lane - j];
        s += (int)c[j];
      }
      int incl = s;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      const int excl = incl - s;  // keys in higher digits than this lane's
      if (excl < krem && krem <= incl) {
        int above = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (above < krem && krem <= above + (int)c[j]) {
            sh[0] = 255 - 8 * lane - j;
            sh[1] = above;
          }
          above += (int)c[j];
        }
      }
    }
    __syncthreads();
    const Key digit = (Key)sh[0];
    krem -= sh[1];
    prefix |= digit << shift;
    pmask |= (Key)0xFF << shift;
    __syncthreads();
  }
  *gt = k - krem;
  return prefix;
}

// Sum of a warp-uniform value over the warps before this one (and the block total).
__device__ int warp_exclusive_sum(int v, int* sh, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const int x = sh[w];
    before += w < warp ? x : 0;
    all += x;
  }
  __syncthreads();
  *total = all;
  return before;
}

// Ordered emission of the first k keys by (key desc, index asc), given the k-th largest key T
// and take = k - #{key > T} (the number of keys equal to T to keep, lowest index first); all keys
// when all.  emit(rank, i) for the kept i in ascending i, rank = 0, 1, ...  Returns the kept count.
// Warp w owns a contiguous range of 32-key groups; lane j takes key 32 g + j of each group, so
// shared-memory reads are conflict-free and global reads coalesced; ranks come from ballots.
template <typename Key, typename KeyAt, typename Emit>
__device__ int block_emit_ordered(KeyAt key_at, int n, bool all, Key T, int take, Emit emit, int* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned lt = (1u << lane) - 1u;
  const int S = ((n + kWarps * 32 - 1) / (kWarps * 32)) * 32;
  const int w0 = min(n, warp * S), w1 = min(n, w0 + S);
  int nt = 0;
  if (!all)
    for (int b = w0; b < w1; b += 32) {
      const int i = b + lane;
      nt += __popc(__ballot_sync(0xffffffffu, i < w1 && key_at(i) == T));
    }
  int tot = 0;
  const int tie_base = warp_exclusive_sum(nt, sh, &tot);
  int nk = 0, tr = tie_base;
  for (int b = w0; b < w1; b += 32) {
    const int i = b + lane;
    const Key u = (i < w1 && !all) ? key_at(i) : (Key)0;
    const bool tie = i < w1 && !all && u == T;
    const unsigned tb = __ballot_sync(0xffffffffu, tie);
    const bool keep = i < w1 && (all || u > T || (tie && tr + __popc(tb & lt) < take));
    nk += __popc(__ballot_sync(0xffffffffu, keep));
    tr += __popc(tb);
  }
  int kept = 0;
  int pos = warp_exclusive_sum(nk, sh, &kept);
  tr = tie_base;
  for (int b = w0; b < w1; b += 32) {
    const int i = b + lane;
    const Key u = (i < w1 && !all) ? key_at(i) : (Key)0;
    const bool tie = i < w1 && !all && u == T;
    const unsigned tb = __ballot_sync(0xffffffffu, tie);
    const bool keep = i < w1 && (all || u > T || (tie && tr + __popc(tb & lt) < take));
    const unsigned kb = __ballot_sync(0xffffffffu, keep);
    if (keep) emit(pos + __popc(kb & lt), i);
    pos += __popc(kb);
    tr += __popc(tb);
  }
  return kept;
}

// Stable compaction of the first k keys by (key desc, index asc) out of n (k >= n keeps all), the
// threshold found by the block radix select.  Returns the kept count.
template <typename Key, typename KeyAt, typename Emit>
__device__ int block_select_ordered(KeyAt key_at, int n, int k, Emit emit, uint32_t* hist, int* sh) {
  Key T = 0;
  int take = n;
  const bool all = k >= n;
  if (!all) {
    int gt = 0;
    T = block_kth_largest<Key>(key_at, n, k, hist, sh, &gt);
    take = k - gt;
  }
  return block_emit_ordered<Key>(key_at, n, all, T, take, emit, sh + 4);
}

// One warp, keys in registers (n <= 2048, 64 per lane): the k-th largest of n 64-bit keys
// (1 <= k <= n) by bisection on their high 32 bits, then on the low 32 bits of the keys whose
// high half equals the threshold's.  Returns T and sets *gt = #{key > T}.  All lanes must call it.
template <typename KeyAt>
__device__ uint64_t warp_kth_largest64(KeyAt key_at, int n, int k, int* gt) {
  constexpr int V = 64;
  const int lane = threadIdx.x & 31;
  uint32_t v[V];
  uint32_t mn = 0xFFFFFFFFu, mx = 0u;
#pragma unroll
  for (int q = 0; q < V; ++q) {
    const int j = q * 32 + lane;
    v[q] = j < n ? (uint32_t)(key_at(j) >> 32) : 0u;
    if (j < n) { mn = min(mn, v[q]); mx = max(mx, v[q]); }
  }
  mn = __reduce_min_sync(0xffffffffu, mn);
  mx = __reduce_max_sync(0xffffffffu, mx);
  uint64_t lo = mn, hi = (uint64_t)mx + 1;  // #{high >= lo} >= k, #{high >= hi} < k
  while (hi - lo > 1) {
    const uint32_t mid = (uint32_t)(lo + ((hi - lo) >> 1));
    int c = 0;
#pragma unroll
    for (int q = 0; q < V; ++q) c += (q * 32 + lane < n && v[q] >= mid) ? 1 : 0;
    if ((int)__reduce_add_sync(0xffffffffu, (unsigned)c) >= k) lo = mid; else hi = mid;
  }
  const uint32_t th = (uint32_t)lo;
  int g = 0;
#pragma unroll
  for (int q = 0; q < V; ++q) g += (q * 32 + lane < n && v[q] > th) ? 1 : 0;
  g = (int)__reduce_add_sync(0xffffffffu, (unsigned)g);
  const int need = k - g;  // >= 1 keys with high half th
  // Low halves of the keys whose high half is th; the rest drop out of the second bisection.
  bool in[V];
  mn = 0xFFFFFFFFu;
  mx = 0u;
#pragma unroll
  for (int q = 0; q < V; ++q) {
    const int j = q * 32 + lane;
    in[q] = j < n && v[q] == th;
    v[q] = in[q] ? (uint32_t)key_at(j) : 0u;
    if (in[q]) { mn = min(mn, v[q]); mx = max(mx, v[q]); }
  }
  mn = __reduce_min_sync(0xffffffffu, mn);
  mx = __reduce_max_sync(0xffffffffu, mx);
  lo = mn;
  hi = (uint64_t)mx + 1;
  while (hi - lo > 1) {
    const uint32_t mid = (uint32_t)(lo + ((hi - lo) >> 1));
    int c = 0;
#pragma unroll
    for (int q = 0; q < V; ++q) c += (in[q] && v[q] >= mid) ? 1 : 0;
    if ((int)__reduce_add_sync(0xffffffffu, (unsigned)c) >= need) lo = mid; else hi = mid;
  }
  int g2 = 0;
#pragma unroll
  for (int q = 0; q < V; ++q) g2 += (in[q] && v[q] > (uint32_t)lo) ? 1 : 0;
  *gt = g + (int)__reduce_add_sync(0xffffffffu, (unsigned)g2);
  return ((uint64_t)th << 32) | (uint32_t)lo;
}

// Block-wide: emit(rank, i) for every i in [0, n) with key_at(i) >= LB, in ascending i; returns
// the count.  Warp-contiguous ranges of 32-key groups, ranks from ballots.
template <typename Key, typename KeyAt, typename Emit>
__device__ int block_filter_ordered(KeyAt key_at, int n, Key LB, Emit emit, int* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned lt = (1u << lane) - 1u;
  const int S = ((n + kWarps * 32 - 1) / (kWarps * 32)) * 32;
  const int w0 = min(n, warp * S), w1 = min(n, w0 + S);
  int nk = 0;
  for (int b = w0; b < w1; b += 32) {
    const int i = b + lane;
    nk += __popc(__ballot_sync(0xffffffffu, i < w1 && key_at(i) >= LB));
  }
  int total = 0;
  int pos = warp_exclusive_sum(nk, sh, &total);
  for (int b = w0; b < w1; b += 32) {
    const int i = b + lane;
    const bool keep = i < w1 && key_at(i) >= LB;
    const unsigned kb = __ballot_sync(0xffffffffu, keep);
    if (keep) emit(pos + __popc(kb & lt), i);
    pos += __popc(kb);
  }
  return total;
}

// ---------------------------------------------------------------------------
// fc_gather
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads) fc_gather_kernel(DecodeParams p, const void* Kc, void* Kfc, int pos0,
                                                             int npos) {
  const int W = 2 * p.nfc;          // columns of a compact row
  const int G8 = W / 8;             // 16-byte groups per compact row
  const size_t items = (size_t)p.B * p.Hkv * npos * G8;
  for (size_t it = (size_t)blockIdx.x * kThreads + threadIdx.x; it < items; it += (size_t)gridDim.x * kThreads) {
    const int grp = (int)(it % G8);
    size_t r = it / G8;
    const int t = pos0 + (int)(r % npos);
    const int bg = (int)(r / npos);  // b * Hkv + g
    const int g = bg % p.Hkv;
    const __nv_bfloat16* krow = static_cast<const __nv_bfloat16*>(Kc) + ((size_t)bg * p.L + t) * p.D;
    uint16_t v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int c = grp * 8 + e;
      const int dim = c < p.nfc ? p.fc[g * p.nfc + c] : p.fc[g * p.nfc + c - p.nfc] + p.D / 2;
      v[e] = reinterpret_cast<const uint16_t*>(krow)[dim];
    }
    uint4 o;
    o.x = v[0] | ((uint32_t)v[1] << 16);
    o.y = v[2] | ((uint32_t)v[3] << 16);
    o.z = v[4] | ((uint32_t)v[5] << 16);
    o.w = v[6] | ((uint32_t)v[7] << 16);
    reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(Kfc) + ((size_t)bg * p.L + t) * W)[grp] = o;
  }
}

// ---------------------------------------------------------------------------
// tip_chunk: persistent, one or two CTAs per SM, looping over tiles (chunk, b,
// KV head); G = Q heads per KV head, TPS = tokens per thread per slab, NGR =
// groups of 4 keys per thread per chunk.  The chunk's compact key rows stream
// through an NS-stage ring of slabs (ST = 256 TPS tokens) filled by bulk
// copies; the ring runs across tiles, so the next tile's first slabs are in
// flight while this tile's candidates are selected.
// ---------------------------------------------------------------------------
template <int G, int TPS, int NGR>
__global__ void __launch_bounds__(kThreads, G <= 4 ? 2 : 1) tip_chunk_kernel(DecodeParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  constexpr int ST = kThreads * TPS;
  const int W = 2 * p.nfc;
  const int C = p.chunk;
  const int NS = p.nstages;
  const uint32_t SB = (uint32_t)ST * W * 2;                                                // slab bytes
  unsigned char* ring = smem_raw;                                                           // [NS][SB]
  uint16_t* keys = reinterpret_cast<uint16_t*>(ring + (size_t)NS * SB);                   // [G][C]
  float* qd = reinterpret_cast<float*>(keys + (size_t)G * C);                              // [W][G]
  __shared__ __align__(8) uint64_t bars[4];
  __shared__ int scratch[128];
  __shared__ int lost;

  const int tid = threadIdx.x;
  const int ntiles = p.nchunks * p.B * p.Hkv;
  const __nv_bfloat16* kfc_all = static_cast<const __nv_bfloat16*>(p.Kfc);
  auto slabs_of = [&](int tile) {
    const int n = min(C, p.L - (tile % p.nchunks) * C);
    return (n + ST - 1) / ST;
  };
  // Producer state (thread 0): next (tile, slab) to copy and the stage it goes to.
  int ptile = blockIdx.x, pslab = 0, issued = 0;
  auto issue_next = [&]() {
    if (ptile >= ntiles) return;
    const int chunk = ptile % p.nchunks, bg = ptile / p.nchunks;
    const int n = min(C, p.L - chunk * C);
    const int rows = min(ST, n - pslab * ST);
    const __nv_bfloat16* src = kfc_all + ((size_t)bg * p.L + (size_t)chunk * C + (size_t)pslab * ST) * W;
    const int stg = issued % NS;
    arm_and_load((uint32_t)__cvta_generic_to_shared(&bars[stg]), (uint32_t)__cvta_generic_to_shared(ring + (size_t)stg * SB),
                 src, (uint32_t)rows * W * 2);
    ++issued;
    if (++pslab == slabs_of(ptile)) {
      pslab = 0;
      ptile += gridDim.x;
    }
  };
  if (tid == 0) {
    lost = 0;
    for (int st = 0; st < NS; ++st)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"((uint32_t)__cvta_generic_to_shared(&bars[st]))
                   : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int st = 0; st < NS; ++st) issue_next();
  }
  __syncthreads();

  int consumed = 0;
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const int chunk = tile % p.nchunks, bg = tile / p.nchunks;
    const int b = bg / p.Hkv, g = bg % p.Hkv;
    const int t0 = chunk * C;
    const int n = min(C, p.L - t0);
    const int nsl = (n + ST - 1) / ST;

    // The group's query values on the dominant dims, column-major: qd[c * G + head].
    for (int e = tid; e < G * W; e += kThreads) {
      const int hh = e % G, c = e / G;
      const int dim = c < p.nfc ? p.fc[g * p.nfc + c] : p.fc[g * p.nfc + c - p.nfc] + p.D / 2;
      const __nv_bfloat16* qrow = static_cast<const __nv_bfloat16*>(p.q) + ((size_t)b * p.Hq + g * G + hh) * p.D;
      qd[c * G + hh] = __bfloat162float(qrow[dim]);
    }
    __syncthreads();

    // Filter scores on the tensor cores: per slab, warp w takes 16-token tiles of its share, the
    // compact columns in k-steps of 8 (mma.sync m16n8k8, bf16 in, float32 out; A = tokens x
    // columns straight from the slab, B = columns x heads, heads >= G zero).  The products are
    // exact and the margin (see the top of this file) covers the accumulation's rounding.
    // am: the largest |k| bit patterns of the chunk's compact values seen by this lane (two bf16
    // halves; |x| orders like its bits for finite x).
    uint32_t am = 0u;
    {
      const int lane = tid & 31, warp = tid >> 5, gq = lane >> 2, tq = lane & 3;
      const int KS = W / 8;
      uint32_t qb[16];  // B fragments: {q[8 ks + 2 tq][gq], q[8 ks + 2 tq + 1][gq]} as bf16 pairs
#pragma unroll
      for (int ks = 0; ks < 16; ++ks) {
        qb[ks] = 0u;
        if (ks < KS && gq < G)
          qb[ks] = pack_bf16x2(qd[(8 * ks + 2 * tq) * G + gq], qd[(8 * ks + 2 * tq + 1) * G + gq]);
      }
      constexpr int MT = ST / 16 / kWarps;  // 16-token tiles per warp per slab
      for (int sl = 0; sl < nsl; ++sl, ++consumed) {
        const int stg = consumed % NS;
        if (!wait_parity_bounded((uint32_t)__cvta_generic_to_shared(&bars[stg]), (consumed / NS) & 1)) lost = 1;
        const unsigned char* slab = ring + (size_t)stg * SB;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          const int r0 = (warp * MT + mt) * 16 + gq;  // slab rows r0 and r0 + 8
          const int t0s = sl * ST + r0;               // their tokens in the chunk
          const uint32_t m0 = t0s < n ? 0x7FFF7FFFu : 0u, m1 = t0s + 8 < n ? 0x7FFF7FFFu : 0u;
          float c[4] = {0.f, 0.f, 0.f, 0.f};
          const unsigned char* row0 = slab + (size_t)r0 * (2 * W) + 4 * tq;
          const unsigned char* row1 = row0 + (size_t)8 * (2 * W);
#pragma unroll
          for (int ks = 0; ks < 16; ++ks) {
            if (ks >= KS) break;
            const uint32_t a0 = *reinterpret_cast<const uint32_t*>(row0 + 16 * ks);
            const uint32_t a1 = *reinterpret_cast<const uint32_t*>(row1 + 16 * ks);
            am = __vmaxu2(am, a0 & m0);
            am = __vmaxu2(am, a1 & m1);
            asm volatile(
                "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5}, {%6}, "
                "{%0, %1, %2, %3};"
                : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                : "r"(a0), "r"(a1), "r"(qb[ks]));
          }
          // c = scores of tokens (r0, r0 + 8) x heads (2 tq, 2 tq + 1)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int hh = 2 * tq + (e & 1);
            const int t = t0s + (e >> 1) * 8;
            if (hh < G && t < n) keys[(size_t)hh * C + t] = (uint16_t)(order_key(c[e]) >> 16);
          }
        }
        __syncthreads();  // stage consumed
        if (tid == 0) issue_next();
      }
    }
    {
      const uint32_t a16 = __reduce_max_sync(0xffffffffu, max(am & 0xFFFFu, am >> 16));
      if ((tid & 31) == 0) scratch[64 + (tid >> 5)] = (int)a16;
    }
    __syncthreads();

    // Per head, a lower bound LB of the chunk's k-th largest key, by warp h alone: the maxima
    // of the C / 4 groups of 4 consecutive keys (0 past the end of the chunk), then a bisection
    // over them in registers.  Any value with at least k group maxima at or above it is at most
    // the chunk's k-th largest float32 score (each maximum is a distinct token), so stopping the
    // bisection early still gives a valid bound; the bound is then lowered by twice the float32
    // chain's rounding bound M (see the top of this file), so that no token of the row's top k
    // by exact score is dropped.
    {
      const int lane = tid & 31, warp = tid >> 5;
      constexpr int NGPL = 8 * NGR;  // groups per lane: C / 4 / 32
      if (warp < G) {
        uint32_t LBw = 0u;
        if (p.k <= 32 * NGPL) {
          const uint16_t* hk = keys + (size_t)warp * C;
          uint32_t gm[NGPL];
          uint32_t mn = 0xFFFFFFFFu, mx = 0u;
#pragma unroll
          for (int j = 0; j < NGPL; ++j) {
            const int t = 4 * (j * 32 + lane);
            const uint2 v = *reinterpret_cast<const uint2*>(hk + t);
            const uint32_t m0 = t < n ? (v.x & 0xFFFFu) : 0u, m1 = t + 1 < n ? (v.x >> 16) : 0u;
            const uint32_t m2 = t + 2 < n ? (v.y & 0xFFFFu) : 0u, m3 = t + 3 < n ? (v.y >> 16) : 0u;
            gm[j] = max(max(m0, m1), max(m2, m3));
            mn = min(mn, gm[j]);
            mx = max(mx, gm[j]);
          }
          mn = __reduce_min_sync(0xffffffffu, mn);
          mx = __reduce_max_sync(0xffffffffu, mx);
          uint64_t lo = mn, hi = (uint64_t)mx + 1;  // #{>= lo} >= k, #{>= hi} < k
          for (int it = 0; it < 24 && hi - lo > 1; ++it) {
            const uint32_t mid = (uint32_t)(lo + ((hi - lo) >> 1));
            int c = 0;
#pragma unroll
            for (int j = 0; j < NGPL; ++j) c += gm[j] >= mid ? 1 : 0;
            if ((int)__reduce_add_sync(0xffffffffu, (unsigned)c) >= p.k) lo = mid; else hi = mid;
          }
          LBw = (uint32_t)lo;
          // M = 2^-16 ||q||_1 A + n 2^-126, every operation rounded up; then LB - 2M rounded down.
          float q1 = 0.f;
          for (int c = lane; c < W; c += 32) q1 = __fadd_ru(q1, fabsf(qd[c * G + warp]));
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) q1 = __fadd_ru(q1, __shfl_xor_sync(0xffffffffu, q1, off));
          uint32_t a16 = 0u;
#pragma unroll
          for (int w = 0; w < kWarps; ++w) a16 = max(a16, (uint32_t)scratch[64 + w]);
          const float A = __uint_as_float(a16 << 16);
          const float M = __fadd_ru(__fmul_ru(__fmul_ru(0x1p-16f, q1), A), (float)W * 0x1p-126f);
          // The stored keys are the high 16 bits of the float32 keys (rounded down), so LBw << 16
          // bounds the true keys of those group maxima from below; the lowered bound is rounded
          // down to 16 bits again for the comparison with the stored keys.
          if (LBw > 0u) LBw = order_key(__fsub_rd(key_value(LBw << 16), __fmul_ru(2.f, M))) >> 16;
        }
        if (lane == 0) scratch[warp] = (int)LBw;
      }
      __syncthreads();
    }
    uint32_t LB[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) LB[hh] = (uint32_t)scratch[hh];
    // Candidates in token order (16-bit key at or above the 16-bit bound: a superset of the tokens
    // whose float32 key reaches the bound): warp w scans its contiguous range [w S, w S + S) of the chunk
    // and writes its own segment of each head's slot (token indices); then it computes its
    // candidates' exact scores in float64, all heads together and four candidates per lane at a
    // time so that their compact rows (just streamed, so read from L2) are in flight together;
    // counts per (slot, warp).
    const int bad = lost;
    {
      const int lane = tid & 31, warp = tid >> 5;
      const unsigned lt = (1u << lane) - 1u;
      const int S = C / kWarps;
      const int w0 = min(n, warp * S), w1 = min(n, w0 + S);
      const __nv_bfloat16* kfc_rows = kfc_all + (size_t)bg * p.L * W;
      int cnt[G];
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        const size_t slot = ((size_t)b * p.Hq + g * G + hh) * p.nchunks + chunk;
        int* ci = p.cand_idx + slot * C + (size_t)warp * S;
        const uint16_t* hk = keys + (size_t)hh * C;
        int c = 0;
        for (int b0 = w0; b0 < w1; b0 += 32) {
          const int i = b0 + lane;
          const bool keep = i < w1 && hk[i] >= LB[hh];
          const unsigned kb = __ballot_sync(0xffffffffu, keep);
          if (keep) ci[c + __popc(kb & lt)] = t0 + i;
          c += __popc(kb);
        }
        cnt[hh] = c;
        if (lane == 0) p.cand_count[slot * kWarps + warp] = bad ? 0 : c;
      }
      __syncwarp();
      int tot = 0;
#pragma unroll
      for (int hh = 0; hh < G; ++hh) tot += cnt[hh];
      constexpr int kBatch = 4;
      for (int q0 = 0; q0 < tot; q0 += 32 * kBatch) {
        int hs[kBatch], rs[kBatch];
        uint4 rows[kBatch][4];  // compact rows of up to 32 columns (W <= 32 here; longer rows loop below)
        const int W8 = W / 8;
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          int q = q0 + u * 32 + lane, hh = 0;
          hs[u] = -1;
          if (q < tot) {
#pragma unroll
            for (int h2 = 0; h2 < G; ++h2) {
              if (hs[u] < 0) {
                if (q < cnt[h2]) { hs[u] = h2; rs[u] = q; } else { q -= cnt[h2]; }
              }
            }
            (void)hh;
          }
          if (hs[u] >= 0 && W8 <= 4) {
            const size_t slot = ((size_t)b * p.Hq + g * G + hs[u]) * p.nchunks + chunk;
            const int t = p.cand_idx[slot * C + (size_t)warp * S + rs[u]];
            const uint4* kr = reinterpret_cast<const uint4*>(kfc_rows + (size_t)t * W);
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8)
              if (q8 < W8) rows[u][q8] = __ldg(kr + q8);
          }
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          if (hs[u] < 0) continue;
          const int hh = hs[u];
          const size_t slot = ((size_t)b * p.Hq + g * G + hh) * p.nchunks + chunk;
          double sc = 0.0;
          if (W8 <= 4) {
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8) {
              if (q8 >= W8) break;
              const uint32_t w[4] = {rows[u][q8].x, rows[u][q8].y, rows[u][q8].z, rows[u][q8].w};
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float kv = __uint_as_float((e & 1) ? (w[e >> 1] & 0xFFFF0000u) : (w[e >> 1] << 16));
                sc = fma((double)qd[(q8 * 8 + e) * G + hh], (double)kv, sc);
              }
            }
          } else {
            const int t = p.cand_idx[slot * C + (size_t)warp * S + rs[u]];
            const uint4* kr = reinterpret_cast<const uint4*>(kfc_rows + (size_t)t * W);
            for (int q8 = 0; q8 < W8; ++q8) {
              const uint4 v = __ldg(kr + q8);
              const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float kv = __uint_as_float((e & 1) ? (w[e >> 1] & 0xFFFF0000u) : (w[e >> 1] << 16));
                sc = fma((double)qd[(q8 * 8 + e) * G + hh], (double)kv, sc);
              }
            }
          }
          p.cand_key[slot * C + (size_t)warp * S + rs[u]] = order_key64(sc);
        }
      }
    }
    if (bad && tid == 0) report(p.status, SFA_ERR_TIMEOUT);
    __syncthreads();  // keys / qd free for the next tile
  }
  // After a wait that gave up, let this CTA's copies land (bounded) before it exits.
  if (tid == 0 && lost) {
    for (int st = 0; st < NS && st < issued; ++st) {
      const int uses = (issued - st + NS - 1) / NS;
      wait_parity_bounded((uint32_t)__cvta_generic_to_shared(&bars[st]), (uses - 1) & 1);
    }
  }
}

// ---------------------------------------------------------------------------
// tip_merge: CTA per (b, h).  The chunks' candidates (token order, float64
// keys, counts per warp segment) are staged in shared memory when they fit
// (kMergeSmem); with k <= 256 the least of the 256 threads' maxima is at most
// the k-th largest key (each maximum is a distinct candidate), so only keys at
// or above it survive; the exact k-th largest of the survivors by radix
// select; the first k by (key desc, index asc) are written ascending.  More
// candidates than fit use the same select over global memory.
// ---------------------------------------------------------------------------
constexpr int kMergeSmem = 12288;
constexpr int kMaxChunks = 512;

__global__ void __launch_bounds__(kThreads) tip_merge_kernel(DecodeParams p) {
  extern __shared__ __align__(16) uint32_t msm[];
  __shared__ uint32_t hist[256];
  __shared__ int sh[64];
  const size_t row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nseg = p.nchunks * kWarps;
  const int S = p.chunk / kWarps;
  const uint64_t* ck = p.cand_key + row * p.nchunks * p.chunk;
  const int* ci = p.cand_idx + row * p.nchunks * p.chunk;
  const int* cc = p.cand_count + row * nseg;
  int* out = p.idx + row * p.k;
  int* off = reinterpret_cast<int*>(msm);  // [nseg + 1] prefix of the segment counts
  {
    // block scan of the segment counts, kThreads segments at a time
    int carry = 0;
    for (int base = 0; base < nseg; base += kThreads) {
      const int sidx = base + tid;
      const int v = sidx < nseg ? cc[sidx] : 0;
      int tot = 0;
      int x = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (lane == 31) sh[warp] = x;
      __syncthreads();
      int before = 0;
      for (int w = 0; w < kWarps; ++w) {
        before += w < warp ? sh[w] : 0;
        tot += sh[w];
      }
      if (sidx < nseg) off[sidx] = carry + before + x - v;
      carry += tot;
      __syncthreads();
    }
    if (tid == 0) off[nseg] = carry;
    __syncthreads();
  }
  const int n = off[nseg];
  // flat candidate position -> offset in the slot array (segment by binary search)
  auto locate = [&](int i) -> size_t {
    int lo = 0, hi = nseg;  // off[lo] <= i < off[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (off[mid] <= i) lo = mid; else hi = mid;
    }
    return (size_t)lo * S + (i - off[lo]);
  };
  int kept;
  const int ob = (nseg + 1 + 3) & ~3;  // keys start after the offsets (16-byte aligned)
  if (n <= kMergeSmem) {
    uint64_t* sk = reinterpret_cast<uint64_t*>(msm + ob);  // [n] keys
    int* st = reinterpret_cast<int*>(sk + n);              // [n] token indices
    int* sv = st + n;                                      // [n] survivor positions
    // Flat copy: thread tid takes candidates tid, tid + 256, ... (segment by binary search), four
    // at a time, so that hundreds of independent loads are in flight instead of one segment's.
    for (int i0 = tid; i0 < n; i0 += 4 * kThreads) {
      uint64_t kv[4];
      int iv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * kThreads;
        if (i < n) {
          const size_t at = locate(i);
          kv[u] = __ldg(ck + at);
          iv[u] = __ldg(ci + at);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * kThreads;
        if (i < n) {
          sk[i] = kv[u];
          st[i] = iv[u];
        }
      }
    }
    __syncthreads();
    if (p.k >= n) {
      for (int i = tid; i < n; i += kThreads) out[i] = st[i];
      kept = n;
    } else {
      uint64_t LB = 0u;
      if (p.k <= kThreads) {
        uint64_t m = 0u;
        for (int i = tid; i < n; i += kThreads) m = max(m, sk[i]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = min(m, __shfl_xor_sync(0xffffffffu, m, o));
        __syncthreads();
        if (lane == 0) reinterpret_cast<uint64_t*>(hist)[warp] = m;
        __syncthreads();
        LB = ~0ull;
        for (int w = 0; w < kWarps; ++w) LB = min(LB, reinterpret_cast<const uint64_t*>(hist)[w]);
        __syncthreads();
      }
      int ns = n;
      if (LB > 0u) {
        ns = block_filter_ordered<uint64_t>([&](int i) { return sk[i]; }, n, LB, [&](int r, int i) { sv[r] = i; },
                                            sh + 16);
      } else {
        for (int i = tid; i < n; i += kThreads) sv[i] = i;
      }
      __syncthreads();
      auto key_s = [&](int j) { return sk[sv[j]]; };
      auto emit_s = [&](int r, int j) { out[r] = st[sv[j]]; };
      if (ns <= 2048) {
        // few survivors: one warp finds the k-th largest in registers, no block barriers per step
        if (warp == 0) {
          int gt = 0;
          const uint64_t T = warp_kth_largest64(key_s, ns, p.k, &gt);
          if (lane == 0) {
            reinterpret_cast<uint64_t*>(hist)[0] = T;
            sh[1] = p.k - gt;
          }
        }
        __syncthreads();
        const uint64_t T = reinterpret_cast<const uint64_t*>(hist)[0];
        const int take = sh[1];
        __syncthreads();
        kept = block_emit_ordered<uint64_t>(key_s, ns, false, T, take, emit_s, sh + 4);
      } else {
        kept = block_select_ordered<uint64_t>(key_s, ns, p.k, emit_s, hist, sh);
      }
    }
  } else {
    kept = block_select_ordered<uint64_t>([&](int i) { return __ldg(ck + locate(i)); }, n, p.k,
                                          [&](int r, int i) { out[r] = __ldg(ci + locate(i)); }, hist, sh);
  }
  for (int r = kept + tid; r < p.k; r += kThreads) out[r] = -1;
}

// ---------------------------------------------------------------------------
// fac: CTA per (b, h), 16 warps
// ---------------------------------------------------------------------------
constexpr int kFacWarps = 16;
constexpr int kFacBatch = 8;  // tokens per warp with loads in flight

template <int D>
__global__ void __launch_bounds__(kFacWarps * 32) fac_kernel(DecodeParams p) {
  constexpr int DPL = D / 32;  // dims per lane (4 for d = 128, 2 for d = 64)
  __shared__ float wm[kFacWarps], wl[kFacWarps];
  __shared__ float wacc[kFacWarps][D];
  __shared__ int bad;
  const size_t row = blockIdx.x;
  const int b = (int)(row / p.Hq), h = (int)(row % p.Hq);
  const int g = h / (p.Hq / p.Hkv);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int* list = p.idx + row * p.k;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();

  float q[DPL];
  {
    const __nv_bfloat16* qrow = static_cast<const __nv_bfloat16*>(p.q) + row * D + lane * DPL;
#pragma unroll
    for (int e = 0; e < DPL; ++e) q[e] = __bfloat162float(qrow[e]) * p.scale;
  }
  const __nv_bfloat16* kbase = static_cast<const __nv_bfloat16*>(p.Kc) + (size_t)(b * p.Hkv + g) * p.L * D;
  const __nv_bfloat16* vbase = static_cast<const __nv_bfloat16*>(p.Vc) + (size_t)(b * p.Hkv + g) * p.L * D;
  float m = -INFINITY, l = 0.f, acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;

  for (int base = warp * kFacBatch; base < p.k; base += kFacWarps * kFacBatch) {
    int tok[kFacBatch];
    float kv[kFacBatch][DPL], vv[kFacBatch][DPL];
#pragma unroll
    for (int u = 0; u < kFacBatch; ++u) {
      const int r = base + u;
      int t = r < p.k ? __ldg(list + r) : -1;
      if (t >= p.L || t < -1) {  // out of range (-1 is padding): record, skip the row
        if (lane == 0) bad = 1;
        t = -1;
      }
      tok[u] = t;
      const int ts = t < 0 ? 0 : t;
      const __nv_bfloat16* kr = kbase + (size_t)ts * D + lane * DPL;
      const __nv_bfloat16* vr = vbase + (size_t)ts * D + lane * DPL;
      if constexpr (DPL == 4) {
        const uint2 ku = __ldg(reinterpret_cast<const uint2*>(kr));
        const uint2 vu = __ldg(reinterpret_cast<const uint2*>(vr));
        kv[u][0] = __uint_as_float(ku.x << 16); kv[u][1] = __uint_as_float(ku.x & 0xFFFF0000u);
        kv[u][2] = __uint_as_float(ku.y << 16); kv[u][3] = __uint_as_float(ku.y & 0xFFFF0000u);
        vv[u][0] = __uint_as_float(vu.x << 16); vv[u][1] = __uint_as_float(vu.x & 0xFFFF0000u);
        vv[u][2] = __uint_as_float(vu.y << 16); vv[u][3] = __uint_as_float(vu.y & 0xFFFF0000u);
      } else {
        const uint32_t ku = __ldg(reinterpret_cast<const uint32_t*>(kr));
        const uint32_t vu = __ldg(reinterpret_cast<const uint32_t*>(vr));
        kv[u][0] = __uint_as_float(ku << 16); kv[u][1] = __uint_as_float(ku & 0xFFFF0000u);
        vv[u][0] = __uint_as_float(vu << 16); vv[u][1] = __uint_as_float(vu & 0xFFFF0000u);
      }
    }
#pragma unroll
    for (int u = 0; u < kFacBatch; ++u) {
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < DPL; ++e) s = fmaf(q[e], kv[u][e], s);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      if (tok[u] < 0) continue;  // padding (warp-uniform)
      const float mn = fmaxf(m, s);
      const float f = expf(m - mn), pe = expf(s - mn);
      l = l * f + pe;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] = fmaf(acc[e], f, pe * vv[u][e]);
      m = mn;
    }
  }
  if (lane == 0) { wm[warp] = m; wl[warp] = l; }
#pragma unroll
  for (int e = 0; e < DPL; ++e) wacc[warp][lane * DPL + e] = acc[e];
  __syncthreads();
  if (bad) {
    if (threadIdx.x == 0) report(p.status, SFA_ERR_INDEX);
  }
  if (threadIdx.x < D) {
    const int dd = threadIdx.x;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kFacWarps; ++w) M = fmaxf(M, wm[w]);
    float L = 0.f, o = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kFacWarps; ++w) {
        const float f = wm[w] == -INFINITY ? 0.f : expf(wm[w] - M);
        L += wl[w] * f;
        o += wacc[w][dd] * f;
      }
    }
    const float out = (bad || L == 0.f) ? 0.f : o / L;
    static_cast<__nv_bfloat16*>(p.o)[row * D + dd] = __float2bfloat16_rn(out);
    if (dd == 0 && p.lse != nullptr) p.lse[row] = (bad || L == 0.f) ? -INFINITY : M + logf(L);
  }
}

}  // namespace

// Chunk geometry for a group size and compact row width: C tokens per chunk, TPS tokens per
// thread per slab, NS ring stages; shared memory = NS slabs + G C 16-bit filter keys + the query table.
DecodeGeometry decode_geometry(int group, int nfc) {
  DecodeGeometry d;
  const int W = 2 * nfc;
  d.tps = W <= 32 ? 2 : 1;
  const size_t slab = (size_t)kThreads * d.tps * W * 2;
  // Two CTAs per SM when the keys and a two-stage ring fit in half the shared memory (228 KB per
  // SM, 1 KB reserved per CTA, under 1 KB of static shared memory per CTA).
  size_t budget = 113 * 1024;
  if ((size_t)group * 4096 * 2 + 2 * slab > budget) budget = 200 * 1024;
  d.chunk = 4096;
  while (d.chunk > 1024 && (size_t)group * d.chunk * 2 + 2 * slab > budget) d.chunk /= 2;
  d.nstages = (int)((budget - (size_t)group * d.chunk * 2) / slab);
  d.nstages = d.nstages > 4 ? 4 : d.nstages;
  d.ctas_per_sm = budget < 150 * 1024 ? 2 : 1;
  d.smem = d.nstages * slab + (size_t)group * d.chunk * 2 + (size_t)group * W * 4;
  return d;
}

int decode_max_chunks() { return kMaxChunks; }

cudaError_t launch_fc_gather(const DecodeParams& p, const void* Kc, void* Kfc, int pos0, int npos, cudaStream_t st) {
  const size_t items = (size_t)p.B * p.Hkv * npos * (2 * p.nfc / 8);
  if (items == 0) return cudaSuccess;
  size_t blocks = (items + kThreads - 1) / kThreads;
  if (blocks > (size_t)148 * 16) blocks = (size_t)148 * 16;
  const unsigned grid = (unsigned)blocks;
  fc_gather_kernel<<<grid, kThreads, 0, st>>>(p, Kc, Kfc, pos0, npos);
  return cudaGetLastError();
}

template <int G, int TPS, int NGR>
static cudaError_t launch_tip_chunk_t(const DecodeParams& p, cudaStream_t st) {
  const DecodeGeometry d = decode_geometry(G, p.nfc);
  auto kern = tip_chunk_kernel<G, TPS, NGR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)d.smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int ntiles = p.nchunks * p.B * p.Hkv;
  const int grid = sms * d.ctas_per_sm;
  kern<<<ntiles < grid ? ntiles : grid, kThreads, d.smem, st>>>(p);
  return cudaGetLastError();
}

template <int G>
static cudaError_t launch_tip_chunk(const DecodeParams& p, cudaStream_t st) {
  const bool two = p.tps == 2;
  const bool four = p.chunk == 4096;  // groups of 4 keys per thread: C / 1024
  if (two) return four ? launch_tip_chunk_t<G, 2, 4>(p, st) : (p.chunk == 2048 ? launch_tip_chunk_t<G, 2, 2>(p, st)
                                                                                : launch_tip_chunk_t<G, 2, 1>(p, st));
  return four ? launch_tip_chunk_t<G, 1, 4>(p, st)
              : (p.chunk == 2048 ? launch_tip_chunk_t<G, 1, 2>(p, st) : launch_tip_chunk_t<G, 1, 1>(p, st));
}

cudaError_t launch_decode_select(const DecodeParams& p, cudaStream_t st) {
  const int G = p.Hq / p.Hkv;
  cudaError_t e = G == 1 ? launch_tip_chunk<1>(p, st)
                  : G == 2 ? launch_tip_chunk<2>(p, st)
                  : G == 4 ? launch_tip_chunk<4>(p, st)
                           : launch_tip_chunk<8>(p, st);
  if (e != cudaSuccess) return e;
  const size_t msmem = ((size_t)p.nchunks * kWarps + 8 + (size_t)4 * kMergeSmem) * sizeof(uint32_t);
  e = cudaFuncSetAttribute(tip_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)msmem);
  if (e != cudaSuccess) return e;
  tip_merge_kernel<<<p.B * p.Hq, kThreads, msmem, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_decode_attn(const DecodeParams& p, cudaStream_t st) {
  if (p.D == 128)
    fac_kernel<128><<<p.B * p.Hq, kFacWarps * 32, 0, st>>>(p);
  else
    fac_kernel<64><<<p.B * p.Hq, kFacWarps * 32, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace sfa
