// Decode-side estimate -> exact attention ("FASA: Frequency-aware Sparse
// Attention" §2B): one query token per (batch, Q head) against a KV cache.
//
//   fc_gather      compact copy K_fc [B, Hkv, L, 2 nfc] of the dominant rotary
//                  pairs of the rotated key cache (low dims, then partners);
//                  run once over the cache, then per appended token range.
//   tip_chunk      Token Importance Predictor, persistent (one or two CTAs per
//                  SM) over tiles (chunk of C tokens, b, KV head): the chunk's
//                  K_fc rows stream through a bulk-copy ring once for all Q
//                  heads of the group (a ninth warp refills each stage as soon
//                  as the eight consumer warps release it); each token's score is first taken on
//                  the tensor cores in float32 (a filter), then per head a lower bound
//                  of the chunk's k-th largest score (from group maxima),
//                  lowered by twice the filter's error bound M, and the tokens
//                  at or above it (token order, per warp segment) as one word
//                  each: 16-bit filter key << 16 | offset in the chunk; M is
//                  recorded per (row, chunk).
//   tip_merge      CTA per (b, h): the candidate words staged in shared memory,
//                  the k-th largest filter key found by bisection and the
//                  candidates bounded again with it, the survivors' exact
//                  scores recomputed in float64 from the compact rows and
//                  ranked (key desc, index asc); ascending index list, -1
//                  padded (a radix select with scores recomputed on the fly
//                  when the candidates do not fit).
//   fac            Focused Attention Computation: CTA per (b, h), 16 warps (8
//                  when the rows fill two CTAs per SM); each warp gathers the
//                  K / V rows of its share of the kept tokens (sixteen tokens'
//                  loads in flight per lane, their indices loaded once and
//                  broadcast), float32 online softmax, warps merged through
//                  shared memory.
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
// The same order without merging the zeros (-0 keys just below +0): for the filter keys, whose
// bounds are always lowered by a positive margin first.
__device__ __forceinline__ uint32_t order_key_signed_zero(float f) {
  const uint32_t u = __float_as_uint(f);
  return u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u);
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
__global__ void __launch_bounds__(kThreads + 32, G <= 4 ? 2 : 1) tip_chunk_kernel(DecodeParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  constexpr int ST = kThreads * TPS;
  const int W = 2 * p.nfc;
  const int C = p.chunk;
  const int NS = p.nstages;
  const uint32_t SB = (uint32_t)ST * W * 2;                                                // slab bytes
  unsigned char* ring = smem_raw;                                                           // [NS][SB]
  uint16_t* keys = reinterpret_cast<uint16_t*>(ring + (size_t)NS * SB);                   // [G][C]
  float* qd = reinterpret_cast<float*>(keys + (size_t)G * C);                              // [W][G]
  __shared__ __align__(8) uint64_t bars[4];   // stage filled (one arrival + the copy's bytes)
  __shared__ __align__(8) uint64_t ebars[4];  // stage consumed (one arrival per consumer warp)
  __shared__ int scratch[128];
  __shared__ int lost;

  const int tid = threadIdx.x;
  const int ntiles = p.nchunks * p.B * p.Hkv;
  const __nv_bfloat16* kfc_all = static_cast<const __nv_bfloat16*>(p.Kfc);
  // Producer state (thread 0): the next (chunk, group, slab) to copy, advanced by the grid size
  // without divisions, and the stage it goes to.
  // This CTA's tiles: a contiguous range (consecutive chunks of one (b, KV head), mostly), the
  // ranges as even as the grid allows.
  const int per_cta = ntiles / (int)gridDim.x, extra = ntiles % (int)gridDim.x;
  const int t_begin = (int)blockIdx.x * per_cta + min((int)blockIdx.x, extra);
  const int t_end = t_begin + per_cta + ((int)blockIdx.x < extra ? 1 : 0);
  int ptile = t_begin, pchunk = t_begin % p.nchunks, pbg = t_begin / p.nchunks, pslab = 0, issued = 0;
  int pn = min(C, p.L - pchunk * C);  // tokens of the producer's chunk
  auto issue_next = [&]() {
    if (ptile >= t_end) return;
    const int rows = min(ST, pn - pslab * ST);
    const __nv_bfloat16* src = kfc_all + ((size_t)pbg * p.L + (size_t)pchunk * C + (size_t)pslab * ST) * W;
    const int stg = issued % NS;
    arm_and_load((uint32_t)__cvta_generic_to_shared(&bars[stg]), (uint32_t)__cvta_generic_to_shared(ring + (size_t)stg * SB),
                 src, (uint32_t)rows * W * 2);
    ++issued;
    if (++pslab * ST >= pn) {
      pslab = 0;
      ++ptile;
      if (++pchunk == p.nchunks) {
        pchunk = 0;
        ++pbg;
      }
      pn = min(C, p.L - pchunk * C);
    }
  };
  if (tid == 0) {
    lost = 0;
    for (int st = 0; st < NS; ++st) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"((uint32_t)__cvta_generic_to_shared(&bars[st]))
                   : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"((uint32_t)__cvta_generic_to_shared(&ebars[st])),
                   "r"(kWarps)
                   : "memory");
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // Warp 8 is the producer: it refills each stage as soon as the eight consumer warps have
  // released it, so no consumer waits on a copy being issued.  The consumers synchronise among
  // themselves on named barrier 1 from here on.
  if (tid >= kThreads) {
    if (tid == kThreads) {
      while (ptile < t_end) {
        const int i = issued;
        if (i >= NS &&
            !wait_parity_bounded((uint32_t)__cvta_generic_to_shared(&ebars[i % NS]), ((i / NS) - 1) & 1))
          lost = 1;
        issue_next();
      }
    }
    return;
  }
  auto consumers_sync = [] { asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory"); };

  int consumed = 0;
  // The bound carried to the next chunk of the same rows (warp h keeps head h's): the raw k-th
  // group maximum of the run's first chunk and that chunk's margin.
  int run_bg = -1;
  uint32_t run_lb = 0u;
  float run_m = 0.f;
  for (int tile = t_begin; tile < t_end; ++tile) {
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
    consumers_sync();

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
        // Fragment rows gq and gq + 8 of tile mt take slab rows r0 and r0 + 1, so that a lane's two
        // tokens are adjacent and their keys of one head go out in one word; the tiles' k-steps are
        // interleaved so that their mma chains overlap.
        const int rb = warp * MT * 16 + 2 * gq;  // tile 0's r0
        const unsigned char* rowb = ring + (size_t)stg * SB + (size_t)rb * (2 * W) + 4 * tq;
        uint32_t m0[MT], m1[MT];
        float c[MT][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          const int t0s = sl * ST + rb + 16 * mt;
          m0[mt] = t0s < n ? 0x7FFF7FFFu : 0u;
          m1[mt] = t0s + 1 < n ? 0x7FFF7FFFu : 0u;
          c[mt][0] = c[mt][1] = c[mt][2] = c[mt][3] = 0.f;
        }
#pragma unroll
        for (int ks = 0; ks < 16; ++ks) {
          if (ks >= KS) break;
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            const unsigned char* row0 = rowb + (size_t)(16 * mt) * (2 * W) + 16 * ks;
            const uint32_t a0 = *reinterpret_cast<const uint32_t*>(row0);
            const uint32_t a1 = *reinterpret_cast<const uint32_t*>(row0 + 2 * W);
            am = __vmaxu2(am, a0 & m0[mt]);
            am = __vmaxu2(am, a1 & m1[mt]);
            asm("mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5}, {%6}, "
                "{%0, %1, %2, %3};"
                : "+f"(c[mt][0]), "+f"(c[mt][1]), "+f"(c[mt][2]), "+f"(c[mt][3])
                : "r"(a0), "r"(a1), "r"(qb[ks]));
          }
        }
        // c[mt] = scores of tokens (t0s, t0s + 1) x heads (2 tq, 2 tq + 1); past the end of the chunk
        // the second token's key is left for the readers to mask
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          const int t0s = sl * ST + rb + 16 * mt;
          if (t0s < n) {
            if (2 * tq < G)
              *reinterpret_cast<uint32_t*>(keys + (size_t)(2 * tq) * C + t0s) =
                  __byte_perm(order_key_signed_zero(c[mt][0]), order_key_signed_zero(c[mt][2]), 0x7632);
            if (2 * tq + 1 < G)
              *reinterpret_cast<uint32_t*>(keys + (size_t)(2 * tq + 1) * C + t0s) =
                  __byte_perm(order_key_signed_zero(c[mt][1]), order_key_signed_zero(c[mt][3]), 0x7632);
          }
        }
        __syncwarp();  // stage consumed by this warp
        if ((tid & 31) == 0)
          asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(
                           (uint32_t)__cvta_generic_to_shared(&ebars[stg]))
                       : "memory");
      }
    }
    {
      const uint32_t a16 = __reduce_max_sync(0xffffffffu, max(am & 0xFFFFu, am >> 16));
      if ((tid & 31) == 0) scratch[64 + (tid >> 5)] = (int)a16;
    }
    consumers_sync();

    // Per head, a lower bound LB of the chunk's k-th largest key, by warp h alone: the maxima
    // of the C / 4 groups of 4 consecutive keys (0 past the end of the chunk), then a bisection
    // over them in registers.  Any value with at least k group maxima at or above it is at most
    // the chunk's k-th largest float32 score (each maximum is a distinct token), so stopping the
    // bisection early still gives a valid bound; the bound is then lowered by twice the float32
    // chain's rounding bound M (see the top of this file), so that no token of the row's top k
    // by exact score is dropped.  A bound found in one chunk holds for the whole row: the next
    // chunks of the same rows in this CTA's range reuse it (lowered by that chunk's margin plus
    // their own) instead of searching again.
    {
      const int lane = tid & 31, warp = tid >> 5;
      constexpr int NGPL = 8 * NGR;  // groups per lane: C / 4 / 32
      if (warp < G) {
        // M = 2^-16 ||q||_1 A + n 2^-126, every operation rounded up (also recorded for the merge).
        float q1 = 0.f;
        for (int c = lane; c < W; c += 32) q1 = __fadd_ru(q1, fabsf(qd[c * G + warp]));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) q1 = __fadd_ru(q1, __shfl_xor_sync(0xffffffffu, q1, off));
        uint32_t a16 = 0u;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) a16 = max(a16, (uint32_t)scratch[64 + w]);
        const float A = __uint_as_float(a16 << 16);
        const float M = __fadd_ru(__fmul_ru(__fmul_ru(0x1p-16f, q1), A), (float)W * 0x1p-126f);
        if (lane == 0) p.cand_margin[((size_t)b * p.Hq + g * G + warp) * p.nchunks + chunk] = M;
        uint32_t LBw = 0u;
        if (p.k <= 32 * NGPL && run_bg == bg) {
          LBw = run_lb >= 0x80u
                    ? order_key(__fsub_rd(key_value(run_lb << 16), __fadd_ru(run_m, M))) >> 16
                    : 0u;
        } else if (p.k <= 32 * NGPL) {
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
          // two maxima per word, counted per halfword
          uint32_t gp[NGPL / 2];
#pragma unroll
          for (int j = 0; j < NGPL / 2; ++j) gp[j] = gm[2 * j] | (gm[2 * j + 1] << 16);
          uint32_t lo = mn, hi = mx + 1;  // #{>= lo} >= k, #{>= hi} < k
          while (hi - lo > 1u) {
            const uint32_t mid = lo + ((hi - lo) >> 1);
            const uint32_t mm = mid | (mid << 16);
            uint32_t a = 0u;
#pragma unroll
            for (int j = 0; j < NGPL / 2; ++j) a += __vsetgeu2(gp[j], mm);
            if ((int)__reduce_add_sync(0xffffffffu, (a & 0xFFFFu) + (a >> 16)) >= p.k) lo = mid; else hi = mid;
          }
          // The stored keys are the high 16 bits of the float32 keys (rounded down), so lo << 16
          // bounds the true keys of those group maxima from below; the lowered bound is rounded
          // down to 16 bits again for the comparison with the stored keys.
          // (Keys under 0x0080 hold no finite score: no bound then.)
          run_lb = lo;
          run_m = M;
          LBw = lo >= 0x80u ? order_key(__fsub_rd(key_value(lo << 16), __fmul_ru(2.f, M))) >> 16 : 0u;
        }
        if (lane == 0) scratch[warp] = (int)LBw;
      }
      consumers_sync();
    }
    uint32_t LB[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) LB[hh] = (uint32_t)scratch[hh];
    // Candidates in token order (16-bit key at or above the 16-bit bound: a superset of the tokens
    // whose float32 key reaches the bound): warp w takes its contiguous range [w S, w S + S) of the
    // chunk, lane l the run of R = S / 32 tokens at w S + l R; per head a lane marks its run's
    // candidates in a bit mask (two keys per compare), a warp scan of the counts places them, and
    // the lane writes its own (16-bit filter key << 16 | token offset in the chunk) into the warp's
    // segment of the head's slot; counts per (slot, warp).  The merge rescores the candidates that
    // survive its own bound.
    const int bad = lost;
    {
      constexpr int R = 4 * NGR;  // tokens per lane: C / 8 warps / 32 lanes
      const int lane = tid & 31, warp = tid >> 5;
      const int S = C / kWarps;
      const int r0 = warp * S + lane * R;                 // the lane's run (8-byte aligned keys)
      const int nv = max(0, min(R, n - r0));              // its tokens inside the chunk
      const uint32_t vmask = nv >= 32 ? 0xFFFFFFFFu : ((1u << nv) - 1u);
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        const uint16_t* hk = keys + (size_t)hh * C + r0;
        uint32_t kk[R / 2];
#pragma unroll
        for (int v = 0; v < R / 4; ++v) {
          const uint2 x = *reinterpret_cast<const uint2*>(hk + 4 * v);
          kk[2 * v] = x.x;
          kk[2 * v + 1] = x.y;
        }
        const uint32_t lb2 = LB[hh] | (LB[hh] << 16);
        uint32_t mask = 0u;
#pragma unroll
        for (int j = 0; j < R / 2; ++j) {
          const uint32_t ge = __vsetgeu2(kk[j], lb2);
          mask |= ((ge & 1u) | ((ge >> 15) & 2u)) << (2 * j);
        }
        mask &= vmask;
        const int cnt = __popc(mask);
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        uint32_t* cw = p.cand + (((size_t)b * p.Hq + g * G + hh) * p.nchunks + chunk) * C + (size_t)warp * S;
        int at = incl - cnt;
        while (mask) {
          const int j = __ffs(mask) - 1;
          mask &= mask - 1u;
          cw[at++] = ((uint32_t)hk[j] << 16) | (uint32_t)(r0 + j);
        }
        const int total = __shfl_sync(0xffffffffu, incl, 31);
        if (lane == 0)
          p.cand_count[(((size_t)b * p.Hq + g * G + hh) * p.nchunks + chunk) * kWarps + warp] = bad ? 0 : total;
      }
    }
    if (bad && tid == 0) report(p.status, SFA_ERR_TIMEOUT);
    run_bg = bg;
    consumers_sync();  // keys / qd free for the next tile
  }
  // After a wait that gave up, let this CTA's copies land (bounded) before it exits: every copy
  // the producer issued completes a phase of its stage's barrier (consumed counts them all).
  if (tid == 0 && lost) {
    for (int st = 0; st < NS && st < consumed; ++st) {
      const int uses = (consumed - st + NS - 1) / NS;
      wait_parity_bounded((uint32_t)__cvta_generic_to_shared(&bars[st]), (uses - 1) & 1);
    }
  }
}

// ---------------------------------------------------------------------------
// tip_merge: CTA per (b, h).  The chunks' candidate words (token order, counts
// per warp segment) are staged in shared memory when they fit (merge_cap <=
// kMergeSmem, set per launch from the number of chunks), a
// warp per segment, and their 16-bit filter keys held in registers.  The k-th
// largest filter key X (a four-way bisection between the least and largest
// key) bounds the row's exact k-th largest score from below by value(X) - M
// (at least k candidates have filter scores >= value(X), each within M of its
// exact score, M = the largest margin of the row's chunks), so only candidates
// whose filter key reaches value(X) - 2 M can be in the top k.  Those
// survivors (in token order) get their exact score in float64 from the
// compact key rows; up to kMergeRank of them are ranked by counting (key desc,
// index asc), up to kMergeExact by a bisection in one warp's registers, more
// by a block radix select with the scores recomputed on the fly, as when the
// candidates do not fit in shared memory.  Output ascending, -1 padded.
// ---------------------------------------------------------------------------
constexpr int kMergeSmem = 12288;                  // candidates staged in shared memory
constexpr int kMergeKeys = kMergeSmem / kThreads;  // filter keys per thread (48)
constexpr int kMergeExact = 2048;                  // survivors rescored into shared memory
constexpr int kMergeRank = 512;                    // survivors ranked by counting
constexpr int kSegBatch = 16;                      // segments a warp stages with their loads in flight
constexpr int kMaxChunks = 512;

__global__ void __launch_bounds__(kThreads, 2) tip_merge_kernel(DecodeParams p) {
  extern __shared__ __align__(16) uint32_t msm[];
  __shared__ uint32_t hist[256];
  __shared__ int sh[64];
  __shared__ int bred[2][3][kWarps];
  __shared__ uint32_t mnx[2][kWarps];
  __shared__ float qf[256];  // this row's query on its KV head's compact columns
  __shared__ float red[kWarps];
  __shared__ int nlose, nabove, nband;
  const size_t row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned lt = (1u << lane) - 1u;
  const int b = (int)(row / p.Hq), h = (int)(row % p.Hq), g = h / (p.Hq / p.Hkv);
  const int W = 2 * p.nfc;
  const int nseg = p.nchunks * kWarps;
  const int S = p.chunk / kWarps;
  const uint32_t* cw = p.cand + row * p.nchunks * p.chunk;
  const int* cc = p.cand_count + row * nseg;
  int* out = p.idx + row * p.k;
  int* off = reinterpret_cast<int*>(msm);  // [nseg + 1] prefix of the segment counts
  if (tid == 0) {
    nlose = 0;
    nabove = 0;
    nband = 0;
  }
  for (int c = tid; c < W; c += kThreads) {
    const int dim = c < p.nfc ? p.fc[g * p.nfc + c] : p.fc[g * p.nfc + c - p.nfc] + p.D / 2;
    qf[c] = __bfloat162float(static_cast<const __nv_bfloat16*>(p.q)[row * p.D + dim]);
  }
  float mg = 0.f;  // the row's largest chunk margin
  for (int c = tid; c < p.nchunks; c += kThreads) mg = fmaxf(mg, p.cand_margin[row * p.nchunks + c]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mg = fmaxf(mg, __shfl_xor_sync(0xffffffffu, mg, o));
  if (lane == 0) red[warp] = mg;
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
  float M = 0.f;
  for (int w = 0; w < kWarps; ++w) M = fmaxf(M, red[w]);
  const int n = off[nseg];
  // segment of candidate position i (binary search over the offsets); token of a word of segment sg
  auto seg_of = [&](int i) -> int {
    int lo = 0, hi = nseg;  // off[lo] <= i < off[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (off[mid] <= i) lo = mid; else hi = mid;
    }
    return lo;
  };
  auto token_of = [&](int sg, uint32_t w) -> int { return (sg / kWarps) * p.chunk + (int)(w & 0xFFFFu); };
  auto token_global = [&](int i) -> int {
    const int sg = seg_of(i);
    return token_of(sg, __ldg(cw + (size_t)sg * S + (i - off[sg])));
  };
  // Exact score of tokens t0 and t1 (t1 < 0: none): the float64 dot product over the compact
  // columns in order, both rows' sixteen-byte groups loaded (four at a time) before the sums.
  const __nv_bfloat16* kfc_rows = static_cast<const __nv_bfloat16*>(p.Kfc) + (size_t)(b * p.Hkv + g) * p.L * W;
  auto rescore2 = [&](int t0, int t1, uint64_t* k0, uint64_t* k1) {
    const uint4* r0 = reinterpret_cast<const uint4*>(kfc_rows + (size_t)t0 * W);
    const uint4* r1 = reinterpret_cast<const uint4*>(kfc_rows + (size_t)(t1 < 0 ? t0 : t1) * W);
    double s0 = 0.0, s1 = 0.0;
    for (int q0 = 0; q0 < W / 8; q0 += 4) {
      uint4 v0[4], v1[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const bool in = q0 + u < W / 8;
        v0[u] = in ? __ldg(r0 + q0 + u) : make_uint4(0u, 0u, 0u, 0u);
        v1[u] = in ? __ldg(r1 + q0 + u) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (q0 + u >= W / 8) break;
        const uint32_t a[4] = {v0[u].x, v0[u].y, v0[u].z, v0[u].w};
        const uint32_t c[4] = {v1[u].x, v1[u].y, v1[u].z, v1[u].w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const double qv = (double)qf[(q0 + u) * 8 + e];
          const float ka = __uint_as_float((e & 1) ? (a[e >> 1] & 0xFFFF0000u) : (a[e >> 1] << 16));
          const float kc = __uint_as_float((e & 1) ? (c[e >> 1] & 0xFFFF0000u) : (c[e >> 1] << 16));
          s0 = fma(qv, (double)ka, s0);
          s1 = fma(qv, (double)kc, s1);
        }
      }
    }
    *k0 = order_key64(s0);
    *k1 = order_key64(s1);
  };
  auto rescore = [&](int t) -> uint64_t {
    uint64_t k0, k1;
    rescore2(t, -1, &k0, &k1);
    return k0;
  };
  int kept;
  const int ob = (nseg + 1 + 3) & ~3;  // arrays start after the offsets (16-byte aligned)
  const int cap = p.merge_cap;
  if (n <= cap) {
    uint64_t* gk = reinterpret_cast<uint64_t*>(msm + ob);  // [kMergeExact] survivors' exact keys
    int* stok = reinterpret_cast<int*>(gk + kMergeExact);   // [kMergeExact] survivors' tokens
    int* sv = stok + kMergeExact;                            // [n] survivor positions (then losers)
    int* wc = sv + cap;                                      // [kMergeKeys][kWarps] counts
    uint32_t* sc = reinterpret_cast<uint32_t*>(wc + kMergeKeys * kWarps);  // [n] candidate words
    // Warp w stages segments kSegBatch at a time (w kSegBatch + 8 kSegBatch j ...): lane l takes words
    // 2 l and 2 l + 1 of each segment in one load (a segment starts 8-byte aligned and both words
    // lie in its slots), all of the batch's loads issued before any store; words past 64 one by one.
    for (int s0 = warp * kSegBatch; s0 < nseg; s0 += kWarps * kSegBatch) {
      uint2 kv[kSegBatch];
#pragma unroll
      for (int u = 0; u < kSegBatch; ++u) {
        const int sg = s0 + u;
        const int cnt = sg < nseg ? off[sg + 1] - off[sg] : 0;
        kv[u] = 2 * lane < cnt ? __ldg(reinterpret_cast<const uint2*>(cw + (size_t)sg * S) + lane) : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kSegBatch; ++u) {
        const int sg = s0 + u;
        const int base = sg < nseg ? off[sg] : 0;
        const int cnt = sg < nseg ? off[sg + 1] - base : 0;
        if (2 * lane < cnt) sc[base + 2 * lane] = kv[u].x;
        if (2 * lane + 1 < cnt) sc[base + 2 * lane + 1] = kv[u].y;
        for (int j = 64 + lane; j < cnt; j += 32) sc[base + j] = __ldg(cw + (size_t)sg * S + j);
      }
    }
    __syncthreads();
    if (p.k >= n) {
      for (int i = tid; i < n; i += kThreads) out[i] = token_of(seg_of(i), sc[i]);
      kept = n;
    } else {
      // Filter keys in registers, candidate i = tid + kThreads q, two per word (0 past the end).
      uint32_t kp[kMergeKeys / 2];
      uint32_t kmin = 0xFFFFu, kmax = 0u;
#pragma unroll
      for (int q2 = 0; q2 < kMergeKeys / 2; ++q2) {
        const int i0 = 2 * q2 * kThreads + tid, i1 = i0 + kThreads;
        const uint32_t a = i0 < n ? sc[i0] >> 16 : 0u, c = i1 < n ? sc[i1] >> 16 : 0u;
        kp[q2] = a | (c << 16);
        if (i0 < n) { kmin = min(kmin, a); kmax = max(kmax, a); }
        if (i1 < n) { kmin = min(kmin, c); kmax = max(kmax, c); }
      }
      kmin = __reduce_min_sync(0xffffffffu, kmin);
      kmax = __reduce_max_sync(0xffffffffu, kmax);
      if (lane == 0) {
        mnx[0][warp] = kmin;
        mnx[1][warp] = kmax;
      }
      __syncthreads();
      // X = the k-th largest filter key: #{key >= lo} >= k > #{key >= hi}, the span cut in four per
      // step (a threshold of 0 counts every candidate; keys past the end are 0 and never count
      // against a threshold >= 1).
      uint32_t lo = 0xFFFFu, hi = 0u;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        lo = min(lo, mnx[0][w]);
        hi = max(hi, mnx[1][w]);
      }
      hi += 1u;
      for (int it = 0; hi - lo > 1u; ++it) {
        const uint32_t span = hi - lo;
        const uint32_t m1 = lo + (span >> 2), m2 = lo + (span >> 1), m3 = lo + ((3u * span) >> 2);
        const uint32_t t1 = m1 | (m1 << 16), t2 = m2 | (m2 << 16), t3 = m3 | (m3 << 16);
        uint32_t a1 = 0u, a2 = 0u, a3 = 0u;  // per-halfword counts (at most kMergeKeys / 2 each)
#pragma unroll
        for (int q2 = 0; q2 < kMergeKeys / 2; ++q2) {
          a1 += __vsetgeu2(kp[q2], t1);
          a2 += __vsetgeu2(kp[q2], t2);
          a3 += __vsetgeu2(kp[q2], t3);
        }
        const uint32_t c1 = __reduce_add_sync(0xffffffffu, (a1 & 0xFFFFu) + (a1 >> 16));
        const uint32_t c2 = __reduce_add_sync(0xffffffffu, (a2 & 0xFFFFu) + (a2 >> 16));
        const uint32_t c3 = __reduce_add_sync(0xffffffffu, (a3 & 0xFFFFu) + (a3 >> 16));
        if (lane == 0) {
          bred[it & 1][0][warp] = (int)c1;
          bred[it & 1][1][warp] = (int)c2;
          bred[it & 1][2][warp] = (int)c3;
        }
        __syncthreads();
        int s1 = 0, s2 = 0, s3 = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
          s1 += bred[it & 1][0][w];
          s2 += bred[it & 1][1][w];
          s3 += bred[it & 1][2][w];
        }
        if (m1 == 0u) s1 = n;
        if (s3 >= p.k) {
          lo = m3;
        } else if (s2 >= p.k) {
          lo = m2;
          hi = m3;
        } else if (s1 >= p.k) {
          lo = m1;
          hi = m2;
        } else {
          hi = m1;
        }
      }
      // Survivors: filter key >= thr (keys under 0x0080 hold no finite score: no bound then),
      // compacted in candidate order from per-(q, warp) ballot counts.
      const uint32_t X = lo;
      const uint32_t thr = X >= 0x80u ? order_key(__fsub_rd(key_value(X << 16), __fmul_ru(2.f, M))) >> 16 : 0u;
      const uint32_t tt = thr | (thr << 16);
      auto survives = [&](int q) {
        const uint32_t ge = __vsetgeu2(kp[q >> 1], tt);
        return ((q & 1) ? (ge >> 16) : (ge & 0xFFFFu)) != 0u && q * kThreads + tid < n;
      };
#pragma unroll
      for (int q = 0; q < kMergeKeys; ++q) {
        const unsigned kb = __ballot_sync(0xffffffffu, survives(q));
        if (lane == 0) wc[q * kWarps + warp] = __popc(kb);
      }
      __syncthreads();
      if (warp == 0) {
        constexpr int PL = kMergeKeys * kWarps / 32;  // counts per lane
        int v[PL];
        int sum = 0;
#pragma unroll
        for (int e = 0; e < PL; ++e) {
          v[e] = wc[lane * PL + e];
          sum += v[e];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        int run = incl - sum;
#pragma unroll
        for (int e = 0; e < PL; ++e) {
          wc[lane * PL + e] = run;
          run += v[e];
        }
        if (lane == 31) sh[0] = incl;
      }
      __syncthreads();
      const int ns = sh[0];
#pragma unroll
      for (int q = 0; q < kMergeKeys; ++q) {
        const bool keep = survives(q);
        const unsigned kb = __ballot_sync(0xffffffffu, keep);
        if (keep) sv[wc[q * kWarps + warp] + __popc(kb & lt)] = q * kThreads + tid;
      }
      __syncthreads();
      // The survivors' tokens and exact keys (the first kMergeExact), two per thread at a time.
      const int nr = min(ns, kMergeExact);
      for (int j0 = tid; j0 < nr; j0 += 2 * kThreads) {
        const int j1 = j0 + kThreads;
        const int i0 = sv[j0];
        const int t0 = token_of(seg_of(i0), sc[i0]);
        int t1 = -1;
        if (j1 < nr) {
          const int i1 = sv[j1];
          t1 = token_of(seg_of(i1), sc[i1]);
        }
        uint64_t k0, k1;
        rescore2(t0, t1, &k0, &k1);
        stok[j0] = t0;
        gk[j0] = k0;
        if (j1 < nr) {
          stok[j1] = t1;
          gk[j1] = k1;
        }
      }
      __syncthreads();
      auto emit_s = [&](int r, int j) { out[r] = stok[j]; };
      if (ns <= kMergeRank) {
        // The band: with X the k-th largest filter key, at least k candidates have exact scores
        // >= v_lo = value(X) - M, and fewer than k have exact scores >= v_hi = value(X + 1) + M
        // (such a score means a filter score >= value(X + 1), i.e. a key above X).  So survivors
        // scoring >= v_hi are all kept, those below v_lo all dropped, and only the band between is
        // ranked, for the k - (number above) places left.  Checked at run time (counts and the
        // key range); otherwise every survivor is ranked.
        bool band = X >= 0x80u && X < 0xFF80u;
        uint64_t klo = 0ull, khi = 0ull;
        if (band) {
          klo = order_key64((double)__fsub_rd(key_value(X << 16), M));
          khi = order_key64((double)__fadd_ru(key_value((X + 1u) << 16), M));
          for (int j = tid; j < ns; j += kThreads) {
            const uint64_t e = gk[j];
            if (e >= khi) atomicAdd(&nabove, 1);
            else if (e >= klo) {
              const int t = atomicAdd(&nband, 1);
              if (t < kMergeKeys * kWarps) wc[t] = j;
            }
          }
        }
        __syncthreads();
        const int na = nabove, nb = nband;
        band = band && na < p.k && na + nb >= p.k && nb <= kMergeKeys * kWarps;
        if (band) {
          // rank within the band (key desc, position asc); the band's last ones and everything
          // below it are the losers
          const int left = p.k - na;
          for (int t = tid; t < nb; t += kThreads) {
            const int j = wc[t];
            const uint64_t e = gk[j];
            int r = 0;
            for (int u = 0; u < nb; ++u) {
              const int j2 = wc[u];
              const uint64_t e2 = gk[j2];
              r += (e2 > e || (e2 == e && j2 < j)) ? 1 : 0;
            }
            if (r >= left) sv[atomicAdd(&nlose, 1)] = j;
          }
          for (int j = tid; j < ns; j += kThreads)
            if (gk[j] < klo) sv[atomicAdd(&nlose, 1)] = j;
        } else {
          // rank of survivor j = #{i : key_i > key_j, or key_i == key_j and i < j} (survivors are in
          // token order): warp w ranks eight survivors at a time, lanes splitting the i range two
          // keys per step, and records those ranked k or later (the ns - k losers); a kept
          // survivor's place in the output is j minus the losers before it
          constexpr int RJ = 8;
          for (int j0 = warp * RJ; j0 < ns; j0 += kWarps * RJ) {
            uint64_t kj[RJ];
            int r[RJ];
#pragma unroll
            for (int u = 0; u < RJ; ++u) {
              kj[u] = gk[min(j0 + u, ns - 1)];
              r[u] = 0;
            }
            for (int i = lane; i < ns; i += 64) {
              const int i2 = i + 32;
              const uint64_t ka = gk[i], kb = i2 < ns ? gk[i2] : 0ull;  // 0: no finite score's key
#pragma unroll
              for (int u = 0; u < RJ; ++u) {
                r[u] += (ka > kj[u] || (ka == kj[u] && i < j0 + u)) ? 1 : 0;
                r[u] += (kb > kj[u] || (kb == kj[u] && i2 < j0 + u)) ? 1 : 0;
              }
            }
            int rr = 0;
#pragma unroll
            for (int u = 0; u < RJ; ++u) {
              const int t = (int)__reduce_add_sync(0xffffffffu, (unsigned)r[u]);
              if (lane == u) rr = t;
            }
            if (lane < RJ && j0 + lane < ns && rr >= p.k) sv[atomicAdd(&nlose, 1)] = j0 + lane;
          }
        }
        __syncthreads();
        const int L = nlose;
        for (int j = tid; j < ns; j += kThreads) {
          int below = 0;
          bool lose = false;
          for (int e = 0; e < L; ++e) {
            const int x = sv[e];
            below += x < j ? 1 : 0;
            lose = lose || x == j;
          }
          if (!lose) out[j - below] = stok[j];
        }
        kept = ns - L;
      } else if (ns <= kMergeExact) {
        // one warp finds the k-th largest exact key in registers, no block barriers per step
        if (warp == 0) {
          int gt = 0;
          const uint64_t T = warp_kth_largest64([&](int j) { return gk[j]; }, ns, p.k, &gt);
          if (lane == 0) {
            reinterpret_cast<uint64_t*>(hist)[0] = T;
            sh[1] = p.k - gt;
          }
        }
        __syncthreads();
        const uint64_t T = reinterpret_cast<const uint64_t*>(hist)[0];
        const int take = sh[1];
        __syncthreads();
        kept = block_emit_ordered<uint64_t>([&](int j) { return gk[j]; }, ns, false, T, take, emit_s, sh + 4);
      } else {
        auto tok = [&](int j) { const int i = sv[j]; return token_of(seg_of(i), sc[i]); };
        kept = block_select_ordered<uint64_t>([&](int j) { return rescore(tok(j)); }, ns, p.k,
                                              [&](int r, int j) { out[r] = tok(j); }, hist, sh);
      }
    }
  } else {
    kept = block_select_ordered<uint64_t>([&](int i) { return rescore(token_global(i)); }, n, p.k,
                                          [&](int r, int i) { out[r] = token_global(i); }, hist, sh);
  }
  for (int r = kept + tid; r < p.k; r += kThreads) out[r] = -1;
}

// ---------------------------------------------------------------------------
// fac: CTA per (b, h), 16 or 8 warps
// ---------------------------------------------------------------------------
constexpr int kFacBatch = 16;  // tokens per warp with loads in flight

template <int D, int kFacWarps>
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
    // The batch's token indices (lane u < kFacBatch loads index base + u), broadcast, then all
    // the batch's K / V row slices loaded before any is used.
    int tl = -1;
    if (lane < kFacBatch && base + lane < p.k) {
      tl = __ldg(list + base + lane);
      if (tl >= p.L || tl < -1) {  // out of range (-1 is padding): record, skip the row
        bad = 1;
        tl = -1;
      }
    }
    int tok[kFacBatch];
    uint2 ku[kFacBatch], vu[kFacBatch];  // this lane's DPL bf16 of the token's K and V rows
#pragma unroll
    for (int u = 0; u < kFacBatch; ++u) {
      tok[u] = __shfl_sync(0xffffffffu, tl, u);
      const int ts = tok[u] < 0 ? 0 : tok[u];
      const __nv_bfloat16* kr = kbase + (size_t)ts * D + lane * DPL;
      const __nv_bfloat16* vr = vbase + (size_t)ts * D + lane * DPL;
      if constexpr (DPL == 4) {
        ku[u] = __ldg(reinterpret_cast<const uint2*>(kr));
        vu[u] = __ldg(reinterpret_cast<const uint2*>(vr));
      } else {
        ku[u] = make_uint2(__ldg(reinterpret_cast<const uint32_t*>(kr)), 0u);
        vu[u] = make_uint2(__ldg(reinterpret_cast<const uint32_t*>(vr)), 0u);
      }
    }
#pragma unroll
    for (int u = 0; u < kFacBatch; ++u) {
      float kv[DPL], vv[DPL];
      kv[0] = __uint_as_float(ku[u].x << 16); kv[1] = __uint_as_float(ku[u].x & 0xFFFF0000u);
      vv[0] = __uint_as_float(vu[u].x << 16); vv[1] = __uint_as_float(vu[u].x & 0xFFFF0000u);
      if constexpr (DPL == 4) {
        kv[2] = __uint_as_float(ku[u].y << 16); kv[3] = __uint_as_float(ku[u].y & 0xFFFF0000u);
        vv[2] = __uint_as_float(vu[u].y << 16); vv[3] = __uint_as_float(vu[u].y & 0xFFFF0000u);
      }
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < DPL; ++e) s = fmaf(q[e], kv[e], s);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      if (tok[u] < 0) continue;  // padding (warp-uniform)
      const float mn = fmaxf(m, s);
      const float f = expf(m - mn), pe = expf(s - mn);
      l = l * f + pe;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] = fmaf(acc[e], f, pe * vv[e]);
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
  kern<<<ntiles < grid ? ntiles : grid, kThreads + 32, d.smem, st>>>(p);
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
  // offsets, survivors' keys and tokens, survivor positions, compaction counts, candidate words
  // Candidate capacity: all of them for a few chunks (about k + 10% per chunk), so that two or three
  // CTAs share an SM when there are many rows; the full kMergeSmem otherwise.
  DecodeParams q = p;
  q.merge_cap = p.nchunks <= 8 ? 4096 : kMergeSmem;
  const size_t msmem = ((size_t)p.nchunks * kWarps + 4 + (size_t)3 * kMergeExact + q.merge_cap +
                        (size_t)kMergeKeys * kWarps + q.merge_cap) * sizeof(uint32_t);
  e = cudaFuncSetAttribute(tip_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)msmem);
  if (e != cudaSuccess) return e;
  tip_merge_kernel<<<p.B * p.Hq, kThreads, msmem, st>>>(q);
  return cudaGetLastError();
}

// 16 warps per row while the rows fill fewer than two CTAs per SM, else 8 (two CTAs per SM).
cudaError_t launch_decode_attn(const DecodeParams& p, cudaStream_t st) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int rows = p.B * p.Hq;
  const bool many = rows >= 2 * sms;
  if (p.D == 128) {
    if (many) fac_kernel<128, 8><<<rows, 256, 0, st>>>(p);
    else fac_kernel<128, 16><<<rows, 512, 0, st>>>(p);
  } else {
    if (many) fac_kernel<64, 8><<<rows, 256, 0, st>>>(p);
    else fac_kernel<64, 16><<<rows, 512, 0, st>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace sfa
