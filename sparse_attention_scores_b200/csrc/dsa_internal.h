// Host-side launchers of the DSA kernels (internal to libdsa; not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/dsa.h"
#include "dsa_common.cuh"

namespace dsa {

// Wall-time limit of every bounded device-side wait, in nanoseconds.  One
// second by default; the environment variable DSA_WAIT_LIMIT_NS overrides it
// (read once), which lets a test force the time-out path.
uint64_t wait_limit_ns();
// Test hook (environment variable DSA_DEBUG_STALL, read once): a kernel id
// (1 = indexer, 3 = sparse MLA) whose CTAs first wait on a barrier that
// nothing arrives at, so that the bounded wait runs out and the kernel takes
// its error path.  0 (the default) disables it.
int debug_stall();
// Fixed limit used while draining copies/MMAs in flight on the error path.
constexpr uint64_t kDrainLimitNs = 1000000000ull;

int device_sm_count();

// Sets a kernel's function attribute (e.g. its dynamic shared-memory opt-in)
// on the current device, skipping the call when the same value is already set
// for this (device, kernel, attribute).  Attributes belong to the device's
// copy of the kernel, so a process that drives several GPUs sets them on
// each.  Callers opt kernels into the device's maximum dynamic shared memory,
// one value per kernel.  Thread-safe.
cudaError_t func_attr_once(const void *kernel, cudaFuncAttribute attr, int value);

// Host-side argument checks shared by the entry points (dsa_api.cu).
dsa_status_t check_dims_common(const dsa_dims_t *d);
dsa_status_t check_mla_dims(const dsa_dims_t &d);
dsa_status_t check_cache(const dsa_cache_t *c, const dsa_dims_t &d);

// 2-D bf16 tensor map over `rows` rows of `cols` elements (row pitch cols * 2
// bytes) with a box of box_cols x box_rows and a 128- (aw = 128) or 64-byte
// (aw = 64) swizzle.  Returns false when the driver entry point is missing or
// rejects the request.
bool make_map_2d_u8(CUtensorMap *map, const void *base, uint64_t cols, uint64_t rows,
                    uint32_t box_cols, uint32_t box_rows, int aw);
bool make_map_2d(CUtensorMap *map, const void *base, uint64_t cols, uint64_t rows,
                 uint32_t box_cols, uint32_t box_rows, int aw);
// [d2][d1][d0] elements of esize bytes (2: bf16, 4: fp32), row strides s1, s2
// bytes; boxes b0 x b1 x b2; 128-byte swizzle (b0 * esize == 128) or none
bool make_map_3d(CUtensorMap *map, const void *base, int esize, uint64_t d0, uint64_t d1,
                 uint64_t d2, uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2,
                 bool swizzle);

// Remember a failed CUDA call of this thread (its error and where it came
// from) for dsa_last_cuda_error(); returns err.
cudaError_t note_cuda_error(cudaError_t err, const char *where);

// Launch `kernel` on `stream` with programmatic stream serialization (the
// kernel calls griddep_wait() before its first dependent read), optionally
// as clusters of cluster_x CTAs.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, unsigned cluster_x, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  const cudaError_t err = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  return err == cudaSuccess ? err : note_cuda_error(err, "kernel launch");
}
size_t device_max_smem_optin();
size_t device_smem_per_sm();

struct IndexerLaunch {
  const uint16_t *q_idx;
  const float *w;
  const uint16_t *k_pages;
  const uint8_t *k8_pages = nullptr;  // E4M3 keys instead of k_pages (with k_scale)
  const float *k_scale = nullptr;     // per physical key row
  const uint8_t *q8 = nullptr;        // K8: E4M3 query terms [2][n_q][H_I][D_I] (w = scaled weights)
  const int32_t *seq_lens;
  const int32_t *block_table;
  float *scores;
  int64_t ld;
  int n_q, H_I, D_I, causal, q_pos0;
  int num_seqs, max_pages, num_pages, max_seq_len;
  DevStatus *status;
  // bf16 keys only: a copy of aux_bytes (a multiple of 16, both ends 16-byte
  // aligned) from aux_src (device-addressable, e.g. mapped host memory) to
  // aux_dst, done by a spare warp of every CTA while the keys are scanned;
  // complete when the indexer grid is
  const void *aux_src = nullptr;
  void *aux_dst = nullptr;
  size_t aux_bytes = 0;
};
dsa_status_t launch_indexer(const IndexerLaunch &a, cudaStream_t stream);
// the E4M3 query terms [2][n_q][H_I][D_I] and scaled weights [n_q][H_I] of the FP8-key indexer
dsa_status_t launch_q8_prep(const uint16_t *q_idx, const float *w, uint8_t *q8, float *w8,
                            int n_q, int H_I, int D_I, cudaStream_t stream);

struct TopkLaunch {
  const float *scores;
  int64_t ld;
  int n_q;
  const int32_t *valid_len;
  int causal_base;
  int k;
  int32_t *idx;
  int max_len;  // host upper bound on any row's length
  DevStatus *status;
};
dsa_status_t launch_topk(const TopkLaunch &a, cudaStream_t stream);

// several device-addressable buffers copied by one kernel (host-buffer step)
constexpr int kMaxCopyPieces = 8;
struct CopyPiece {
  const void *src;
  void *dst;
  uint64_t bytes;
};
struct CopyList {
  CopyPiece piece[kMaxCopyPieces];
  int n;
};
dsa_status_t launch_copy_pieces(const CopyList &l, cudaStream_t stream);

struct AppendLaunch {
  const uint16_t *k_new;
  const uint16_t *lat_new;
  uint16_t *k_pages;
  uint16_t *lat_pages;
  const int32_t *seq_lens;
  const int32_t *block_table;
  int n_q, D_I, W, causal, q_pos0, max_pages, num_pages;
  DevStatus *status;
};
dsa_status_t launch_append(const AppendLaunch &a, cudaStream_t stream);

struct AbsorbLaunch {
  bool project;          // false: q_abs = q_nope . W_UK (+ rope); true: v_out = o_lat . W_UV
  const uint16_t *x;     // q_nope [n, H, K] bf16 (absorb)
  const float *xf;       // o_lat  [n, H, K] fp32 (project)
  const uint16_t *rope;  // q_rope [n, H, P] (absorb, may be null when P == 0)
  const uint16_t *w;     // W_UK [H, K, M] or W_UV [H, K, M] bf16
  uint16_t *out_bf16;    // q_abs [n, H, M + P]
  float *out_f32;        // v_out [n, H, M]
  int n, H, K, M, P;
  DevStatus *status;
};
dsa_status_t launch_absorb(const AbsorbLaunch &a, cudaStream_t stream);

// context-parallel decode (cp.cu)
dsa_status_t launch_cp_candidates(const float *scores, int64_t ld, int n_q, const int32_t *idx_local,
                                  int k, const int32_t *offsets, float *cand_s, int32_t *cand_i,
                                  cudaStream_t s);
dsa_status_t launch_cp_pack(const float *all_s, int R, int n_q, int k, int64_t ld, float *packed,
                            int32_t *vlen, cudaStream_t s);
dsa_status_t launch_cp_select(const int32_t *pos, const int32_t *all_i, int R, int n_q, int k,
                              const int32_t *my_off, const int32_t *my_len, int32_t *gidx,
                              int32_t *own, cudaStream_t s);
dsa_status_t launch_cp_merge(const float *outs, const float *lses, int R, int n_q, int H, int dv,
                             float *out, float *lse, cudaStream_t s);

struct MlaLaunch {
  const uint16_t *q;
  const uint16_t *latent;
  const uint8_t *latent8 = nullptr;   // E4M3 latent rows instead of `latent` (with lat_scale)
  const float *lat_scale = nullptr;   // one fp32 scale per physical latent row
  const int32_t *idx;
  const int32_t *seq_lens;
  const int32_t *block_table;
  float *out;
  float *lse;
  int n_q, H, R, P, topk, causal, q_pos0;
  int max_pages, num_pages;
  float scale;
  void *scratch;        // partial results when the keys are split over CTAs
  size_t scratch_bytes;
  DevStatus *status;
  // 1 when q is known to be complete before the kernel preceding this one in
  // the stream started (the fused forward): the query tile is then loaded
  // before waiting on that kernel, overlapping its tail
  int early_q = 0;
  // 1: the pipelined kernel whatever the batch (its small batches merge their
  // splits inside clusters, with no partials in scratch)
  int force_pipe = 0;
};
// Number of key splits the launcher uses, and the scratch bytes it needs
// (enough for either latent format).
int mla_num_splits(int n_q, int topk);
size_t mla_scratch_bytes(int n_q, int topk, int R);
// the scratch bytes of the pipelined kernel alone (force_pipe)
size_t mla_pipe_scratch_bytes(int n_q, int topk, int R);
dsa_status_t launch_mla(const MlaLaunch &a, cudaStream_t stream);
// Kernels launch_mla launches for these shapes on the current device (1 or 2;
// lat8: FP8 latent rows).
int mla_launch_count(int n_q, int topk, int R, int P, bool lat8 = false);

}  // namespace dsa
