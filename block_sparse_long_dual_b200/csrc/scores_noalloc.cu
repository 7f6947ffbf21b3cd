// sfa_block_scores_noalloc: sfa_block_scores with its scratch in a fixed
// device array owned by this library, for callers that cannot allocate.
//
// The scratch is a file-scope __device__ array.  Host code cannot use the
// array's name as a device address (on the host it names a stand-in object),
// so the device address is looked up once per device with
// cudaGetSymbolAddress, with that device current, and then passed to the same
// kernels sfa_block_scores launches.
#include <cuda_runtime.h>

#include <mutex>

#include "sfa.h"

namespace {

constexpr size_t kScratchBytes = SFA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scores_scratch[kScratchBytes];

std::mutex g_lock;
void* g_scratch_ptr[kMaxDevices];  // set once a lookup on that device succeeded

// The scratch array's device address on the current device `dev`, looked up on first use.  Only a
// successful lookup is cached, so a lookup that failed (for instance a first call made while the
// stream was being captured, which is refused before any lookup) is retried by the next call.
void* scratch_address(int dev, cudaStream_t stream) {
  std::lock_guard<std::mutex> guard(g_lock);
  if (g_scratch_ptr[dev] != nullptr) return g_scratch_ptr[dev];
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone) return nullptr;
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_scores_scratch) != cudaSuccess) return nullptr;
  g_scratch_ptr[dev] = ptr;
  return ptr;
}

}  // namespace

extern "C" sfa_status sfa_block_scores_noalloc(const sfa_shape* shape, const void* Q, const void* K,
                                               const sfa_rope* rope, int band_split, int block, unsigned flags,
                                               void* Q_rot, void* K_rot, float* probs, void* stream) {
  const size_t need = sfa_block_scores_workspace(shape, block);
  if (need == 0)  // invalid shape: let the full validation report the precise status
    return sfa_block_scores(shape, Q, K, rope, band_split, block, flags, Q_rot, K_rot, probs, nullptr, 0, stream);
  if (need > kScratchBytes) return SFA_ERR_WORKSPACE;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return SFA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SFA_ERR_UNSUPPORTED;
  void* scratch = scratch_address(dev, static_cast<cudaStream_t>(stream));
  if (scratch == nullptr) return SFA_ERR_CUDA;
  // Every scratch region (block means, energies, temperatures) is fully written by the
  // kernels before it is read, so nothing left by an earlier call needs clearing.
  return sfa_block_scores(shape, Q, K, rope, band_split, block, flags, Q_rot, K_rot, probs, scratch,
                          kScratchBytes, stream);
}
