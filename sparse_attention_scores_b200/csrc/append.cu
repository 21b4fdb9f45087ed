// Cache append: the new tokens' index keys and latent rows into the paged
// caches, the step in front of the indexer.
//
// ("Self-contained GLM-5 serving stack: Just Vx kernels compiled to PTX",
// file list: absorbed MLA decode over compressed request-local KV, which the
// engine grows by one compressed row per token; "GLM on an A100, in Vx",
// "The model": one latent vector per token, plus the indexer's key.)
//
// One warp per new token: 16-byte loads of its index key (2 D_I bytes) and its
// latent row (2 (R + P) bytes), 16-byte stores into the token's page slot.
// Pure data movement; its roofline is the copy bandwidth.
#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kThreads = 256;
constexpr int kRowsPerCta = kThreads / 32;

struct AppendParams {
  const uint4 *k_new;
  const uint4 *lat_new;
  uint4 *k_pages;
  uint4 *lat_pages;
  const int32_t *seq_lens;
  const int32_t *block_table;
  int n_q;
  int kw, lw;  // 16-byte pieces of one key row / one latent row
  int causal, q_pos0, max_pages, num_pages;
  DevStatus *status;
};

__global__ void __launch_bounds__(kThreads) append_kernel(const AppendParams p) {
  // the new rows, the block table and seq_lens may come from earlier work
  griddep_wait();
  griddep_launch_dependents();
  const int r = blockIdx.x * kRowsPerCta + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (r >= p.n_q) return;
  const int seq = p.causal ? 0 : r;
  const int pos = p.causal ? p.q_pos0 + r : p.seq_lens[r] - 1;
  if (pos < 0 || pos >= p.max_pages * kPageSize) {
    if (lane == 0) report(p.status, kErrBadIndex, (kKernAppend << 24) | (r & 0xFFFF));
    return;
  }
  const int page = p.block_table[static_cast<int64_t>(seq) * p.max_pages + pos / kPageSize];
  if (page < 0 || page >= p.num_pages) {
    if (lane == 0) report(p.status, kErrBadPage, (kKernAppend << 24) | (r & 0xFFFF));
    return;
  }
  const int64_t slot = static_cast<int64_t>(page) * kPageSize + pos % kPageSize;
  const uint4 *ks = p.k_new + static_cast<int64_t>(r) * p.kw;
  const uint4 *ls = p.lat_new + static_cast<int64_t>(r) * p.lw;
  uint4 *kd = p.k_pages + slot * p.kw;
  uint4 *ld = p.lat_pages + slot * p.lw;
  for (int i = lane; i < p.kw; i += 32) kd[i] = ks[i];
  for (int i = lane; i < p.lw; i += 32) ld[i] = ls[i];
}

}  // namespace

dsa_status_t launch_append(const AppendLaunch &a, cudaStream_t stream) {
  AppendParams p;
  p.k_new = reinterpret_cast<const uint4 *>(a.k_new);
  p.lat_new = reinterpret_cast<const uint4 *>(a.lat_new);
  p.k_pages = reinterpret_cast<uint4 *>(a.k_pages);
  p.lat_pages = reinterpret_cast<uint4 *>(a.lat_pages);
  p.seq_lens = a.seq_lens;
  p.block_table = a.block_table;
  p.n_q = a.n_q;
  p.kw = a.D_I * 2 / 16;
  p.lw = a.W * 2 / 16;
  p.causal = a.causal;
  p.q_pos0 = a.q_pos0;
  p.max_pages = a.max_pages;
  p.num_pages = a.num_pages;
  p.status = a.status;
  const unsigned grid = static_cast<unsigned>((a.n_q + kRowsPerCta - 1) / kRowsPerCta);
  if (launch_pdl(append_kernel, dim3(grid), dim3(kThreads), 0, stream, 1, p) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

}  // namespace dsa
