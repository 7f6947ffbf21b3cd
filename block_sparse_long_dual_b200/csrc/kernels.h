// Internal launch interface between the C-ABI host layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace sfa {

struct RopePoolParams {
  const void* Q;
  const void* K;
  void* Qr;
  void* Kr;
  const float* cos;
  const float* sin;
  int apply;      // rotate (else Q, K are already rotated)
  int write_rot;  // write the rotated copies
  double* qbar;
  double* kbar;
  double* energy;
  int B, Hq, Hkv, L, block, nb;
  int band_pairs;  // rotary pairs in band H (d/2 with a single band)
};

struct TauParams {
  const double* energy;
  double* tau;
  int B, Hq, Hkv, L, nb;
  unsigned flags;
};

struct ScoreParams {
  const double* qbar;
  const double* kbar;
  const double* tau;
  const double* energy;  // per-block energies (SFA_BLOCK_TAU)
  float* probs;  // may be null when the selection is fused
  int B, Hq, Hkv, nb, block;
  int band_pairs;
  // fused selection (counts != null): the rule of SelectParams
  int* counts;
  int* idx;
  int kmax;
  int k;
  double mass;
  unsigned flags;
};

struct SelectParams {
  const float* probs;
  int* counts;
  int* idx;
  int B, Hq, nb, kmax;
  int k;        // >= 0: top-k; < 0: mass
  double mass;
  unsigned flags;
};

struct AttnParams {
  const void* Q;
  const void* K;
  const void* V;
  const int* counts;
  const int* idx;
  void* O;
  float* lse;
  int* status;
  const float* rope_cos;  // non-null: Q is pre-RoPE and is rotated on load with these [L, d/2] tables
  const float* rope_sin;
  int B, Hq, Hkv, L, block, nb, kmax;
  int causal;
  float scale;  // softmax scale (natural-log units)
};

// Decode step (one query token per (b, h) against a KV cache of L tokens).
struct DecodeParams {
  const void* q;     // [B, Hq, D] bf16, rotated at the query's position
  const void* Kfc;   // [B, Hkv, L, 2 nfc] bf16 compact dominant-pair keys
  const void* Kc;    // [B, Hkv, L, D] bf16 rotated key cache
  const void* Vc;    // [B, Hkv, L, D] bf16 value cache
  uint32_t* cand;      // [B * Hq, nchunks, chunk] each chunk's candidates in token order per warp segment:
                       // 16-bit filter key << 16 | token offset in the chunk
  int* cand_count;     // [B * Hq, nchunks, 8] per warp segment of each chunk
  float* cand_margin;  // [B * Hq, nchunks] error bound of the chunk's filter scores
  int* idx;          // [B, Hq, k]
  void* o;           // [B, Hq, D] bf16
  float* lse;        // [B, Hq] (nullable)
  int* status;
  int B, Hq, Hkv, L, D, nfc, k, chunk, nchunks, tps, nstages;
  int merge_cap;     // candidates a merge CTA stages in shared memory (set at launch)
  float scale;
  uint8_t fc[1024];  // [Hkv][nfc] dominant pair indices
};

cudaError_t launch_rope_pool_energy(const RopePoolParams& p, int dtype, int D, cudaStream_t st);
cudaError_t launch_band_temperature(const TauParams& p, cudaStream_t st);
cudaError_t launch_block_score_softmax(const ScoreParams& p, int D, cudaStream_t st);
size_t score_smem_bytes(int nb, int D, bool band_max);
cudaError_t launch_select(const SelectParams& p, cudaStream_t st);
cudaError_t launch_attn_simt(const AttnParams& p, int dtype, int D, cudaStream_t st);
struct DecodeGeometry {
  int chunk, tps, nstages, ctas_per_sm;
  size_t smem;
};
DecodeGeometry decode_geometry(int group, int nfc);
int decode_max_chunks();
cudaError_t launch_fc_gather(const DecodeParams& p, const void* Kc, void* Kfc, int pos0, int npos, cudaStream_t st);
cudaError_t launch_decode_select(const DecodeParams& p, cudaStream_t st);
cudaError_t launch_decode_attn(const DecodeParams& p, cudaStream_t st);
cudaError_t launch_attn_tcgen05(const AttnParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                const CUtensorMap& tmV, cudaStream_t st);

}  // namespace sfa
