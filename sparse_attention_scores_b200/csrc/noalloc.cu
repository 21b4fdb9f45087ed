// dsa_sparse_mla_decode_noalloc: the sparse MLA decode for callers that
// cannot allocate device memory.  Its scratch is a fixed file-scope device
// array instead of a caller-provided workspace, and it always runs the
// pipelined kernel, whose small batches merge their splits inside clusters
// and so need no partials at all.
#include <math.h>

#include <mutex>

#include "dsa_internal.h"

namespace dsa {
namespace {

// 16 MiB: the status block plus the split partials of, e.g., one row of
// top-8,192 (64 splits, 8.4 MB).  Rows split over the CTAs of one cluster
// (a batch of 32 at top-2,048) or not split at all (as many rows as SMs) need
// no partials.  Every GPU that loads the library holds it until the process
// exits.
constexpr size_t kNoAllocScratchBytes = 16ull << 20;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// In host code `g_noalloc_scratch` names a host-side stand-in, not the device
// array: its device address is looked up once per device, with that device
// current, and cached here.
constexpr int kMaxDev = 64;
void *g_scratch_addr[kMaxDev];
std::once_flag g_scratch_once[kMaxDev];
cudaError_t g_scratch_err[kMaxDev];

void *scratch_address(int dev, dsa_status_t *st) {
  if (dev < 0 || dev >= kMaxDev) {
    *st = DSA_ERR_CUDA;
    return nullptr;
  }
  std::call_once(g_scratch_once[dev], [dev] {
    void *ptr = nullptr;
    g_scratch_err[dev] = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    g_scratch_addr[dev] = (g_scratch_err[dev] == cudaSuccess) ? ptr : nullptr;
  });
  *st = (g_scratch_addr[dev] != nullptr) ? DSA_OK : DSA_ERR_CUDA;
  return g_scratch_addr[dev];
}

bool aligned_to(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" DSA_API dsa_status_t dsa_sparse_mla_decode_noalloc(
    const uint16_t *q, const uint16_t *latent_pages, const dsa_cache_t *cache, const int32_t *idx,
    const dsa_dims_t *dims, float *out, float *lse, dsa_stream_t stream) {
  // the same host checks as dsa_sparse_mla_decode (decode rows only)
  dsa_status_t chk = check_dims_common(dims);
  if (chk != DSA_OK) return chk;
  if (dims->causal != 0) return DSA_ERR_INVALID_ARG;
  if ((chk = check_mla_dims(*dims)) != DSA_OK) return chk;
  if ((chk = check_cache(cache, *dims)) != DSA_OK) return chk;
  const dsa_dims_t &d = *dims;
  if (q == nullptr || latent_pages == nullptr || idx == nullptr || out == nullptr || lse == nullptr)
    return DSA_ERR_INVALID_ARG;
  if (!aligned_to(q, 16) || !aligned_to(latent_pages, 16) || !aligned_to(idx, 4) ||
      !aligned_to(out, 4) || !aligned_to(lse, 4))
    return DSA_ERR_INVALID_ARG;
  const dsa_cache_t &c = *cache;
  // the built-in array holds the status block and the split partials
  const size_t need = sizeof(DevStatus) + mla_pipe_scratch_bytes(d.n_q, d.topk, d.R);
  if (need > kNoAllocScratchBytes) return DSA_ERR_WORKSPACE;
  if (d.n_q == 0) return DSA_OK;

  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSA_ERR_CUDA;
  dsa_status_t st = DSA_OK;
  uint8_t *base = static_cast<uint8_t *>(scratch_address(dev, &st));
  if (st != DSA_OK) return st;
  cudaStream_t s = stream ? reinterpret_cast<cudaStream_t>(stream) : cudaStreamPerThread;
  // the array keeps the previous call's contents: clear the status block
  if (cudaMemsetAsync(base, 0, sizeof(DevStatus), s) != cudaSuccess) return DSA_ERR_CUDA;

  MlaLaunch a;
  a.q = q;
  a.latent = latent_pages;
  a.idx = idx;
  a.seq_lens = c.seq_lens;
  a.block_table = c.block_table;
  a.out = out;
  a.lse = lse;
  a.n_q = d.n_q;
  a.H = d.H;
  a.R = d.R;
  a.P = d.P;
  a.topk = d.topk;
  a.causal = 0;
  a.q_pos0 = 0;
  a.max_pages = c.max_pages;
  a.num_pages = c.num_pages;
  a.scale = d.scale;
  a.scratch = base + sizeof(DevStatus);
  a.scratch_bytes = kNoAllocScratchBytes - sizeof(DevStatus);
  a.status = reinterpret_cast<DevStatus *>(base);
  a.force_pipe = 1;
  return launch_mla(a, s);
}

extern "C" DSA_API dsa_status_t dsa_noalloc_status(dsa_stream_t stream, uint32_t *info) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSA_ERR_CUDA;
  dsa_status_t st = DSA_OK;
  const void *base = scratch_address(dev, &st);
  if (st != DSA_OK) return st;
  cudaStream_t s = stream ? reinterpret_cast<cudaStream_t>(stream) : cudaStreamPerThread;
  DevStatus host;
  if (cudaMemcpyAsync(&host, base, sizeof(host), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return DSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DSA_ERR_CUDA;
  if (info) *info = host.first;
  if (host.flags & kErrTimeout) return DSA_ERR_TIMEOUT;
  if (host.flags != 0u) return DSA_ERR_DEVICE_CHECK;
  return DSA_OK;
}
