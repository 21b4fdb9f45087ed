// Moving one step's small host buffers with one kernel each way.
//
// A copy-engine transfer costs several microseconds of latency however few
// bytes it moves, and the step's per-step inputs and results are tens to
// hundreds of kilobytes in several buffers.  Pinned host memory that the
// device can address (mapped, as page-locked allocations are under unified
// addressing) is read and written here by the SMs directly: every piece of a
// list is spread over many threads with 16-byte accesses where source,
// destination and size allow, so the PCIe round trips overlap.
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kCopyThreads = 256;

__global__ void __launch_bounds__(kCopyThreads) copy_pieces_kernel(const CopyList l) {
  // the previous kernel on the stream may still read a destination or write a source
  griddep_wait();
  griddep_launch_dependents();
  const CopyPiece pc = l.piece[blockIdx.y];
  const uint8_t *src = static_cast<const uint8_t *>(pc.src);
  uint8_t *dst = static_cast<uint8_t *>(pc.dst);
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * kCopyThreads;
  const uint64_t t0 = static_cast<uint64_t>(blockIdx.x) * kCopyThreads + threadIdx.x;
  if (((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst) | pc.bytes) & 15u) == 0) {
    const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
    const uint64_t n = pc.bytes / 16;
    for (uint64_t i = t0; i < n; i += stride) d4[i] = s4[i];
  } else if (((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst) | pc.bytes) & 3u) == 0) {
    const uint32_t *s1 = reinterpret_cast<const uint32_t *>(src);
    uint32_t *d1 = reinterpret_cast<uint32_t *>(dst);
    const uint64_t n = pc.bytes / 4;
    for (uint64_t i = t0; i < n; i += stride) d1[i] = s1[i];
  } else {
    for (uint64_t i = t0; i < pc.bytes; i += stride) dst[i] = src[i];
  }
}

}  // namespace

dsa_status_t launch_copy_pieces(const CopyList &l, cudaStream_t stream) {
  if (l.n <= 0) return DSA_OK;
  if (l.n > kMaxCopyPieces) return DSA_ERR_INVALID_ARG;
  uint64_t most = 0;
  for (int i = 0; i < l.n; ++i) most = most > l.piece[i].bytes ? most : l.piece[i].bytes;
  // enough threads for two 16-byte accesses each on the largest piece
  const uint64_t blocks = (most / 16 + 2 * kCopyThreads - 1) / (2 * kCopyThreads);
  const unsigned gx = static_cast<unsigned>(blocks < 1 ? 1 : (blocks > 1024 ? 1024 : blocks));
  if (launch_pdl(copy_pieces_kernel, dim3(gx, static_cast<unsigned>(l.n)), dim3(kCopyThreads), 0,
                 stream, 1u, l) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

}  // namespace dsa
