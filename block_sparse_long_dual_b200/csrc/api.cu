// C-ABI host layer: argument validation, workspace layout, tensor maps and
// kernel launches on the caller's stream.  Declarations and the contract of
// every entry point are in include/sfa.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "kernels.h"
#include "sfa.h"

using namespace sfa;

namespace {

constexpr int kVersion = 100;  // 0.1.0
constexpr int kMaxBlocks = 2048;
constexpr unsigned kKnownFlags =
    SFA_KEEP_SINK | SFA_NO_CALIB | SFA_SINGLE_BAND | SFA_RELATIVE_CALIB | SFA_BAND_MAX | SFA_BLOCK_TAU;

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Common shape checks; nb_out receives L / block.
sfa_status check_shape(const sfa_shape* s, int block, int* nb_out) {
  if (s == nullptr) return SFA_ERR_INVALID_ARG;
  if (s->dtype != SFA_F32 && s->dtype != SFA_BF16) return SFA_ERR_DTYPE;
  if (s->batch < 1 || s->heads_q < 1 || s->heads_kv < 1 || s->seq_len < 1) return SFA_ERR_SHAPE;
  if (s->head_dim != 64 && s->head_dim != 128) return SFA_ERR_SHAPE;
  if (block != 64 && block != 128) return SFA_ERR_SHAPE;
  if (s->heads_q % s->heads_kv != 0) return SFA_ERR_SHAPE;
  if (s->seq_len % block != 0) return SFA_ERR_SHAPE;
  const int nb = s->seq_len / block;
  if (nb > kMaxBlocks) return SFA_ERR_UNSUPPORTED;
  // Row indices of the [B*H*L, d] views and tile ids must fit in int32.
  const long long rows = (long long)s->batch * s->heads_q * s->seq_len;
  if (rows >= (1LL << 31)) return SFA_ERR_UNSUPPORTED;
  if (nb_out) *nb_out = nb;
  return SFA_OK;
}

struct WsLayout {
  size_t off[4];
  size_t total;
};

WsLayout ws_layout(const sfa_shape* s, int nb) {
  WsLayout w;
  const size_t d = s->head_dim;
  size_t o = 0;
  w.off[0] = o;
  o = align256(o + (size_t)s->batch * s->heads_q * nb * d * sizeof(double));
  w.off[1] = o;
  o = align256(o + (size_t)s->batch * s->heads_kv * nb * d * sizeof(double));
  w.off[2] = o;
  o = align256(o + (size_t)s->batch * (s->heads_q + s->heads_kv) * nb * 4 * sizeof(double));
  w.off[3] = o;
  o = align256(o + (size_t)s->batch * s->heads_q * 2 * sizeof(double));
  w.total = o;
  return w;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda link).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 2D bf16 view [rows, 128] with 64 x 128 boxes and 128-byte swizzle.
bool make_tile_map(CUtensorMap* m, const void* base, uint64_t rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {128, rows};
  const cuuint64_t strides[1] = {128 * 2};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

sfa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SFA_OK : SFA_ERR_CUDA; }

}  // namespace

extern "C" {

int sfa_version(void) { return kVersion; }

const char* sfa_status_string(sfa_status status) {
  switch (status) {
    case SFA_OK: return "ok";
    case SFA_ERR_INVALID_ARG: return "invalid argument";
    case SFA_ERR_SHAPE: return "invalid shape";
    case SFA_ERR_DTYPE: return "unsupported dtype";
    case SFA_ERR_UNSUPPORTED: return "unsupported configuration";
    case SFA_ERR_WORKSPACE: return "workspace missing or too small";
    case SFA_ERR_CUDA: return "CUDA error";
    case SFA_ERR_TIMEOUT: return "device wait timed out";
    case SFA_ERR_INDEX: return "invalid block index list";
  }
  return "unknown status";
}

sfa_status sfa_rope_table(double base, int seq_len, int head_dim, float* cos_out, float* sin_out,
                          void* stream) {
  if (cos_out == nullptr || sin_out == nullptr || !(base > 0.0)) return SFA_ERR_INVALID_ARG;
  if (seq_len < 1 || head_dim < 2 || (head_dim & 1)) return SFA_ERR_SHAPE;
  const int half = head_dim / 2;
  const size_t n = (size_t)seq_len * half;
  std::vector<float> c(n), s(n);
  std::vector<double> theta(half);
  for (int m = 0; m < half; ++m) theta[m] = pow(base, -2.0 * m / head_dim);
  for (int p = 0; p < seq_len; ++p) {
    for (int m = 0; m < half; ++m) {
      const double a = (double)p * theta[m];
      c[(size_t)p * half + m] = (float)cos(a);
      s[(size_t)p * half + m] = (float)sin(a);
    }
  }
  cudaStream_t st = as_stream(stream);
  // Pageable source: the call returns once the host data has been staged.
  if (cudaMemcpyAsync(cos_out, c.data(), n * sizeof(float), cudaMemcpyHostToDevice, st) != cudaSuccess)
    return SFA_ERR_CUDA;
  if (cudaMemcpyAsync(sin_out, s.data(), n * sizeof(float), cudaMemcpyHostToDevice, st) != cudaSuccess)
    return SFA_ERR_CUDA;
  return SFA_OK;
}

size_t sfa_block_scores_workspace(const sfa_shape* shape, int block) {
  int nb = 0;
  if (check_shape(shape, block, &nb) != SFA_OK) return 0;
  return ws_layout(shape, nb).total;
}

sfa_status sfa_workspace_layout(const sfa_shape* shape, int block, size_t offsets[4]) {
  int nb = 0;
  const sfa_status st = check_shape(shape, block, &nb);
  if (st != SFA_OK) return st;
  if (offsets == nullptr) return SFA_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(shape, nb);
  for (int q = 0; q < 4; ++q) offsets[q] = w.off[q];
  return SFA_OK;
}

}  // extern "C"

namespace {

struct FusedSelect {
  int k;
  float mass;
  int* counts;
  int* idx;
  int kmax;
};

// Selection-rule checks shared by sfa_select and sfa_block_scores_select.
sfa_status check_select(int nb, int k, float mass, unsigned flags, const int* counts, const int* idx, int kmax) {
  if (counts == nullptr || idx == nullptr) return SFA_ERR_INVALID_ARG;
  if (flags & ~kKnownFlags) return SFA_ERR_INVALID_ARG;
  const int nforced = (flags & SFA_KEEP_SINK) && nb > 1 ? 2 : 1;
  int need;
  if (k >= 0) {
    need = k + nforced < nb ? k + nforced : nb;
  } else {
    if (!(mass > 0.f && mass <= 1.f)) return SFA_ERR_INVALID_ARG;
    need = nb;
  }
  if (kmax < need || kmax < 1) return SFA_ERR_INVALID_ARG;
  return SFA_OK;
}

sfa_status run_block_scores(const sfa_shape* shape, const void* Q, const void* K, const sfa_rope* rope, int band_split,
                            int block, unsigned flags, void* Q_rot, void* K_rot, float* probs, void* workspace,
                            size_t workspace_bytes, void* stream, const FusedSelect* fused) {
  int nb = 0;
  sfa_status st = check_shape(shape, block, &nb);
  if (st != SFA_OK) return st;
  const int D = shape->head_dim;
  if (Q == nullptr || K == nullptr || rope == nullptr || (probs == nullptr && fused == nullptr))
    return SFA_ERR_INVALID_ARG;
  if (flags & ~kKnownFlags) return SFA_ERR_INVALID_ARG;
  if (band_split < 0 || band_split > D / 2) return SFA_ERR_INVALID_ARG;
  if ((flags & SFA_BLOCK_TAU) && (flags & (SFA_NO_CALIB | SFA_RELATIVE_CALIB))) return SFA_ERR_INVALID_ARG;
  if (fused != nullptr) {
    st = check_select(nb, fused->k, fused->mass, flags, fused->counts, fused->idx, fused->kmax);
    if (st != SFA_OK) return st;
  }
  // Q_rot may be NULL: the rotated Q is then not stored (sfa_block_sparse_attn_rope rotates it on load).
  if (rope->apply && (rope->cos == nullptr || rope->sin == nullptr || K_rot == nullptr))
    return SFA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || (rope->apply && (!aligned16(Q_rot) || !aligned16(K_rot) ||
                                                         !aligned16(rope->cos) || !aligned16(rope->sin))))
    return SFA_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(shape, nb);
  if (workspace == nullptr || workspace_bytes < w.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return SFA_ERR_WORKSPACE;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  cudaStream_t cs = as_stream(stream);
  const int band_pairs = (flags & SFA_SINGLE_BAND) ? D / 2 : band_split;

  RopePoolParams rp;
  rp.Q = Q; rp.K = K; rp.Qr = Q_rot; rp.Kr = K_rot;
  rp.cos = rope->cos; rp.sin = rope->sin;
  rp.apply = rope->apply ? 1 : 0;
  rp.write_rot = rope->apply ? 1 : 0;
  rp.qbar = reinterpret_cast<double*>(ws + w.off[0]);
  rp.kbar = reinterpret_cast<double*>(ws + w.off[1]);
  rp.energy = reinterpret_cast<double*>(ws + w.off[2]);
  rp.B = shape->batch; rp.Hq = shape->heads_q; rp.Hkv = shape->heads_kv;
  rp.L = shape->seq_len; rp.block = block; rp.nb = nb; rp.band_pairs = band_pairs;
  st = cuda_status(launch_rope_pool_energy(rp, shape->dtype, D, cs));
  if (st != SFA_OK) return st;

  TauParams tp;
  tp.energy = rp.energy;
  tp.tau = reinterpret_cast<double*>(ws + w.off[3]);
  tp.B = rp.B; tp.Hq = rp.Hq; tp.Hkv = rp.Hkv; tp.L = rp.L; tp.nb = nb; tp.flags = flags;
  st = cuda_status(launch_band_temperature(tp, cs));
  if (st != SFA_OK) return st;

  ScoreParams sp;
  sp.qbar = rp.qbar; sp.kbar = rp.kbar; sp.tau = tp.tau; sp.energy = rp.energy; sp.probs = probs;
  sp.B = rp.B; sp.Hq = rp.Hq; sp.Hkv = rp.Hkv; sp.nb = nb; sp.block = block; sp.band_pairs = band_pairs;
  sp.counts = fused ? fused->counts : nullptr;
  sp.idx = fused ? fused->idx : nullptr;
  sp.kmax = fused ? fused->kmax : 0;
  sp.k = fused ? fused->k : 0;
  sp.mass = fused ? (double)fused->mass : 0.0;
  sp.flags = flags;
  return cuda_status(launch_block_score_softmax(sp, D, cs));
}

}  // namespace

extern "C" {

sfa_status sfa_block_scores(const sfa_shape* shape, const void* Q, const void* K, const sfa_rope* rope,
                            int band_split, int block, unsigned flags, void* Q_rot, void* K_rot, float* probs,
                            void* workspace, size_t workspace_bytes, void* stream) {
  return run_block_scores(shape, Q, K, rope, band_split, block, flags, Q_rot, K_rot, probs, workspace,
                          workspace_bytes, stream, nullptr);
}

sfa_status sfa_block_scores_select(const sfa_shape* shape, const void* Q, const void* K, const sfa_rope* rope,
                                   int band_split, int block, unsigned flags, int k, float mass, void* Q_rot,
                                   void* K_rot, float* probs, int* counts, int* idx, int kmax, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  const FusedSelect f{k, mass, counts, idx, kmax};
  return run_block_scores(shape, Q, K, rope, band_split, block, flags, Q_rot, K_rot, probs, workspace,
                          workspace_bytes, stream, &f);
}

sfa_status sfa_select(const sfa_shape* shape, int block, const float* probs, int k, float mass, unsigned flags,
                      int* counts, int* idx, int kmax, void* stream) {
  int nb = 0;
  sfa_status st = check_shape(shape, block, &nb);
  if (st != SFA_OK) return st;
  if (probs == nullptr) return SFA_ERR_INVALID_ARG;
  st = check_select(nb, k, mass, flags, counts, idx, kmax);
  if (st != SFA_OK) return st;
  SelectParams p;
  p.probs = probs; p.counts = counts; p.idx = idx;
  p.B = shape->batch; p.Hq = shape->heads_q; p.nb = nb; p.kmax = kmax;
  p.k = k; p.mass = (double)mass; p.flags = flags;
  return cuda_status(launch_select(p, as_stream(stream)));
}

}  // extern "C"

namespace {

sfa_status run_attn(const sfa_shape* shape, int block, const void* Q, const void* K, const void* V,
                    const sfa_rope* rope, const int* counts, const int* idx, int kmax, int causal, float scale,
                    void* O, float* lse, int* status_word, void* stream) {
  int nb = 0;
  sfa_status st = check_shape(shape, block, &nb);
  if (st != SFA_OK) return st;
  if (Q == nullptr || K == nullptr || V == nullptr || counts == nullptr || idx == nullptr || O == nullptr)
    return SFA_ERR_INVALID_ARG;
  if (kmax < 1 || !(isfinite(scale))) return SFA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return SFA_ERR_INVALID_ARG;
  const bool rot = rope != nullptr && rope->apply;
  if (rot && (rope->cos == nullptr || rope->sin == nullptr || !aligned16(rope->cos) || !aligned16(rope->sin)))
    return SFA_ERR_INVALID_ARG;
  const int D = shape->head_dim;
  AttnParams p;
  p.Q = Q; p.K = K; p.V = V; p.counts = counts; p.idx = idx; p.O = O; p.lse = lse; p.status = status_word;
  p.rope_cos = rot ? rope->cos : nullptr;
  p.rope_sin = rot ? rope->sin : nullptr;
  p.B = shape->batch; p.Hq = shape->heads_q; p.Hkv = shape->heads_kv; p.L = shape->seq_len;
  p.block = block; p.nb = nb; p.kmax = kmax; p.causal = causal ? 1 : 0;
  p.scale = scale > 0.f ? scale : (float)(1.0 / sqrt((double)D));
  cudaStream_t cs = as_stream(stream);
  if (shape->dtype == SFA_BF16 && block == 128 && D == 128) {
    CUtensorMap tq, tk, tv;
    const uint64_t rq = (uint64_t)p.B * p.Hq * p.L, rkv = (uint64_t)p.B * p.Hkv * p.L;
    if (!make_tile_map(&tq, Q, rq) || !make_tile_map(&tk, K, rkv) || !make_tile_map(&tv, V, rkv))
      return SFA_ERR_CUDA;
    return cuda_status(launch_attn_tcgen05(p, tq, tk, tv, cs));
  }
  return cuda_status(launch_attn_simt(p, shape->dtype, D, cs));
}

}  // namespace

extern "C" {

sfa_status sfa_block_sparse_attn(const sfa_shape* shape, int block, const void* Q, const void* K, const void* V,
                                 const int* counts, const int* idx, int kmax, int causal, float scale, void* O,
                                 float* lse, int* status_word, void* stream) {
  return run_attn(shape, block, Q, K, V, nullptr, counts, idx, kmax, causal, scale, O, lse, status_word, stream);
}

sfa_status sfa_block_sparse_attn_rope(const sfa_shape* shape, int block, const void* Q, const sfa_rope* rope,
                                      const void* K_rot, const void* V, const int* counts, const int* idx, int kmax,
                                      int causal, float scale, void* O, float* lse, int* status_word,
                                      void* stream) {
  if (rope == nullptr || !rope->apply) return SFA_ERR_INVALID_ARG;
  return run_attn(shape, block, Q, K_rot, V, rope, counts, idx, kmax, causal, scale, O, lse, status_word, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode step
// ---------------------------------------------------------------------------
namespace {

sfa_status check_decode_shape(const sfa_shape* s) {
  if (s == nullptr) return SFA_ERR_INVALID_ARG;
  if (s->dtype != SFA_BF16) return SFA_ERR_DTYPE;
  if (s->batch < 1 || s->heads_q < 1 || s->heads_kv < 1 || s->seq_len < 1) return SFA_ERR_SHAPE;
  if (s->head_dim != 64 && s->head_dim != 128) return SFA_ERR_SHAPE;
  if (s->heads_q % s->heads_kv != 0) return SFA_ERR_SHAPE;
  const int group = s->heads_q / s->heads_kv;
  if (group != 1 && group != 2 && group != 4 && group != 8) return SFA_ERR_UNSUPPORTED;
  if ((long long)s->batch * s->heads_kv * s->seq_len >= (1LL << 31)) return SFA_ERR_UNSUPPORTED;
  return SFA_OK;
}

// Fills the shape fields and the dominant-pair table of p; validates fc.
sfa_status decode_params(const sfa_shape* s, const int* fc, int nfc, DecodeParams* p) {
  sfa_status st = check_decode_shape(s);
  if (st != SFA_OK) return st;
  memset(p, 0, sizeof(*p));
  p->B = s->batch; p->Hq = s->heads_q; p->Hkv = s->heads_kv; p->L = s->seq_len; p->D = s->head_dim;
  const int half = s->head_dim / 2;
  // Without a pair list (sizing, attention) the geometry of the widest list bounds the workspace.
  const DecodeGeometry geo = decode_geometry(s->heads_q / s->heads_kv, fc == nullptr ? half : nfc);
  p->chunk = geo.chunk;
  p->tps = geo.tps;
  p->nstages = geo.nstages;
  p->nchunks = (s->seq_len + p->chunk - 1) / p->chunk;
  if (p->nchunks > decode_max_chunks()) return SFA_ERR_UNSUPPORTED;
  if (fc == nullptr) return nfc == 0 ? SFA_OK : SFA_ERR_INVALID_ARG;
  if (nfc < 4 || nfc > half || nfc % 4 != 0 || s->heads_kv * nfc > (int)sizeof(p->fc)) return SFA_ERR_INVALID_ARG;
  for (int g = 0; g < s->heads_kv; ++g) {
    unsigned long long seen = 0;
    for (int c = 0; c < nfc; ++c) {
      const int m = fc[g * nfc + c];
      if (m < 0 || m >= half || (seen >> m) & 1ull) return SFA_ERR_INVALID_ARG;
      seen |= 1ull << m;
      p->fc[g * nfc + c] = (uint8_t)m;
    }
  }
  p->nfc = nfc;
  return SFA_OK;
}

// Candidate slots: every chunk of every row may keep up to all its tokens.  Sized for the
// largest chunk geometry (4096 tokens) and the most chunks (1024 tokens each), so one
// workspace serves every pair list.
size_t decode_ws_bytes(const DecodeParams& p, int /*k*/) {
  const size_t rows = (size_t)p.B * p.Hq;
  const size_t slots = rows * (((size_t)p.L + 4095) / 4096) * 4096;
  const size_t counts = rows * (((size_t)p.L + 1023) / 1024) * 8;
  const size_t margins = rows * (((size_t)p.L + 1023) / 1024);
  return align256(slots * sizeof(uint32_t)) + align256(counts * sizeof(int)) + align256(margins * sizeof(float));
}

}  // namespace

extern "C" {

size_t sfa_decode_workspace(const sfa_shape* shape, int k) {
  DecodeParams p;
  if (k < 1 || decode_params(shape, nullptr, 0, &p) != SFA_OK) return 0;
  return decode_ws_bytes(p, k);
}

sfa_status sfa_decode_fc_gather(const sfa_shape* shape, const void* K_cache, const int* fc, int nfc, int pos0,
                                int npos, void* K_fc, void* stream) {
  DecodeParams p;
  sfa_status st = decode_params(shape, fc, nfc, &p);
  if (st != SFA_OK) return st;
  if (fc == nullptr || K_cache == nullptr || K_fc == nullptr) return SFA_ERR_INVALID_ARG;
  if (pos0 < 0 || npos < 0 || (long long)pos0 + npos > shape->seq_len) return SFA_ERR_INVALID_ARG;
  if (!aligned16(K_cache) || !aligned16(K_fc)) return SFA_ERR_INVALID_ARG;
  return cuda_status(launch_fc_gather(p, K_cache, K_fc, pos0, npos, as_stream(stream)));
}

sfa_status sfa_decode_select(const sfa_shape* shape, const void* q, const void* K_fc, const int* fc, int nfc, int k,
                             int* idx, void* workspace, size_t workspace_bytes, int* status_word, void* stream) {
  DecodeParams p;
  sfa_status st = decode_params(shape, fc, nfc, &p);
  if (st != SFA_OK) return st;
  if (fc == nullptr || q == nullptr || K_fc == nullptr || idx == nullptr || k < 1) return SFA_ERR_INVALID_ARG;
  if (!aligned16(K_fc)) return SFA_ERR_INVALID_ARG;
  const size_t need = decode_ws_bytes(p, k);
  if (workspace == nullptr || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return SFA_ERR_WORKSPACE;
  const size_t n = (size_t)p.B * p.Hq * p.nchunks * p.chunk;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  p.q = q; p.Kfc = K_fc; p.idx = idx; p.k = k; p.status = status_word;
  const size_t cnts = (size_t)p.B * p.Hq * (((size_t)p.L + 1023) / 1024) * 8;
  p.cand = reinterpret_cast<uint32_t*>(ws);
  p.cand_count = reinterpret_cast<int*>(ws + align256(n * sizeof(uint32_t)));
  p.cand_margin = reinterpret_cast<float*>(ws + align256(n * sizeof(uint32_t)) + align256(cnts * sizeof(int)));
  return cuda_status(launch_decode_select(p, as_stream(stream)));
}

sfa_status sfa_decode_attn(const sfa_shape* shape, const void* q, const void* K_cache, const void* V_cache,
                           const int* idx, int k, float scale, void* o, float* lse, int* status_word, void* stream) {
  DecodeParams p;
  sfa_status st = decode_params(shape, nullptr, 0, &p);
  if (st != SFA_OK) return st;
  if (q == nullptr || K_cache == nullptr || V_cache == nullptr || idx == nullptr || o == nullptr || k < 1)
    return SFA_ERR_INVALID_ARG;
  if (!isfinite(scale)) return SFA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(K_cache) || !aligned16(V_cache)) return SFA_ERR_INVALID_ARG;
  p.q = q; p.Kc = K_cache; p.Vc = V_cache; p.idx = const_cast<int*>(idx); p.k = k;
  p.o = o; p.lse = lse; p.status = status_word;
  p.scale = scale > 0.f ? scale : (float)(1.0 / sqrt((double)shape->head_dim));
  return cuda_status(launch_decode_attn(p, as_stream(stream)));
}

}  // extern "C"

namespace sfa {
cudaError_t launch_bounded_wait_selftest(int* status, uint64_t limit_ns, int arrive, cudaStream_t st);  // selftest.cu
}  // namespace sfa

extern "C" {

sfa_status sfa_selftest_bounded_wait(int* status_word, unsigned limit_ms, int complete, void* stream) {
  if (status_word == nullptr || limit_ms == 0 || limit_ms > 10000) return SFA_ERR_INVALID_ARG;
  return cuda_status(launch_bounded_wait_selftest(status_word, (uint64_t)limit_ms * 1000000ull, complete ? 1 : 0,
                                                  as_stream(stream)));
}

}  // extern "C"
