// Context-parallel decode of one long sequence whose keys are split over
// ranks: the steps around the collectives.
//
// ("GLM on an A100, in Vx", "The model": a context of up to 1,048,576 tokens
// and an exact top-k of 2,048 per query.)  Each rank scores and selects over
// its own key range with the single-device kernels; then
//   candidates  each kept local position becomes a (score, global index) pair
//   select      after an all-gather of every rank's pairs (ranks in key-range
//               order, so the pairs are in ascending global index), the exact
//               global top-k is the top-k of the pairs (the same radix-select
//               kernel, same lower-index tie rule); the kept pairs are
//               compacted to ascending global indices, and each rank marks
//               the ones in its own range as its local positions
//   merge       after every rank attends over its own kept keys and the
//               (out, lse) pairs are all-gathered: the log-sum-exp merge of
//               disjoint key sets
#include <math.h>

#include <algorithm>

#include "dsa_internal.h"

namespace dsa {
namespace {

__global__ void __launch_bounds__(256) cp_candidates_kernel(const float *scores, int64_t ld,
                                                            int n_q, const int32_t *idx_local,
                                                            int k, const int32_t *offsets,
                                                            float *cand_s, int32_t *cand_i) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  if (t >= static_cast<int64_t>(n_q) * k) return;
  const int r = static_cast<int>(t / k);
  const int l = idx_local[t];
  cand_s[t] = (l >= 0) ? scores[static_cast<int64_t>(r) * ld + l] : -INFINITY;
  cand_i[t] = (l >= 0) ? offsets[r] + l : -1;
}

// rank-major [R][n_q][k] scores -> rows [n_q][ld] (ld >= R * k) for the top-k
// kernel, and each row's length R * k
__global__ void __launch_bounds__(256) cp_pack_kernel(const float *all_s, int R, int n_q, int k,
                                                      int64_t ld, float *packed, int32_t *vlen) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  const int64_t per_row = static_cast<int64_t>(R) * k;
  if (t < n_q) vlen[t] = static_cast<int32_t>(per_row);
  if (t >= static_cast<int64_t>(n_q) * per_row) return;
  const int r = static_cast<int>(t / per_row);
  const int64_t c = t - r * per_row;
  const int rank = static_cast<int>(c / k), j = static_cast<int>(c - static_cast<int64_t>(rank) * k);
  packed[static_cast<int64_t>(r) * ld + c] = all_s[(static_cast<int64_t>(rank) * n_q + r) * k + j];
}

// One CTA per row: the kept positions of the packed row (ascending) mapped to
// global indices, pads dropped with order kept, then this rank's own ones
constexpr int kSelThreads = 1024;
__global__ void __launch_bounds__(kSelThreads) cp_select_kernel(
    const int32_t *pos, const int32_t *all_i, int R, int n_q, int k, const int32_t *my_off,
    const int32_t *my_len, int32_t *gidx, int32_t *own) {
  // per warp: kept picks, and kept picks in this rank's range
  __shared__ int warp_tot[2][kSelThreads / 32];
  __shared__ int carry[2];
  griddep_wait();
  griddep_launch_dependents();
  const int r = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int off = my_off[r], len = my_len[r];
  if (tid < 2) carry[tid] = 0;
  __syncthreads();
  for (int base = 0; base < k; base += kSelThreads) {
    const int j = base + tid;
    int g = -1;
    if (j < k) {
      const int p = pos[static_cast<int64_t>(r) * k + j];
      if (p >= 0) {
        const int rank = p / k, slot = p - rank * k;
        if (rank < R) g = all_i[(static_cast<int64_t>(rank) * n_q + r) * k + slot];
      }
    }
    const int v = (g >= 0) ? 1 : 0;
    const int m = (g >= off && g < off + len) ? 1 : 0;  // one of this rank's tokens
    int incl = v, incl_m = m;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      const int ym = __shfl_up_sync(0xffffffffu, incl_m, o);
      if (lane >= o) { incl += y; incl_m += ym; }
    }
    if (lane == 31) { warp_tot[0][warp] = incl; warp_tot[1][warp] = incl_m; }
    __syncthreads();
    if (warp < 2) {
      const int x = warp_tot[warp][lane];
      int wi = x;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += y;
      }
      warp_tot[warp][lane] = wi - x;  // exclusive over warps
    }
    __syncthreads();
    const int dst = carry[0] + warp_tot[0][warp] + incl - v;
    const int dst_m = carry[1] + warp_tot[1][warp] + incl_m - m;
    // the global picks in their global slots; this rank's share compacted to
    // the front of own (local positions, ascending like the global slots)
    if (v) gidx[static_cast<int64_t>(r) * k + dst] = g;
    if (m) own[static_cast<int64_t>(r) * k + dst_m] = g - off;
    __syncthreads();
    if (tid == kSelThreads - 1) {
      carry[0] = dst + v;
      carry[1] = dst_m + m;
    }
    __syncthreads();
  }
  for (int j = carry[0] + tid; j < k; j += kSelThreads) gidx[static_cast<int64_t>(r) * k + j] = -1;
  for (int j = carry[1] + tid; j < k; j += kSelThreads) own[static_cast<int64_t>(r) * k + j] = -1;
}

// out = sum_r exp(lse_r - L) out_r, L = log sum_r exp(lse_r); grid (n_q, H).
// The first warp turns the ranks' lse into normalised weights once; every
// thread then owns columns and reads each rank's value once.
constexpr int kMaxMergeRanks = 1024;
__global__ void __launch_bounds__(128) cp_merge_kernel(const float *outs, const float *lses, int R,
                                                       int n_q, int H, int dv, float *out,
                                                       float *lse) {
  __shared__ float wts[kMaxMergeRanks];
  griddep_wait();
  griddep_launch_dependents();
  const int r = blockIdx.x, h = blockIdx.y, lane = threadIdx.x & 31;
  if (threadIdx.x < 32) {
    float m = -INFINITY;
    for (int q = lane; q < R; q += 32) m = fmaxf(m, lses[(static_cast<int64_t>(q) * n_q + r) * H + h]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float tot = 0.f;
    for (int q = lane; q < R; q += 32) {
      const float l = lses[(static_cast<int64_t>(q) * n_q + r) * H + h];
      const float e = (l == -INFINITY) ? 0.f : expf(l - m);
      wts[q] = e;
      tot += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    const float inv = (tot > 0.f) ? 1.f / tot : 0.f;
    for (int q = lane; q < R; q += 32) wts[q] *= inv;
    if (lane == 0) lse[static_cast<int64_t>(r) * H + h] = (tot > 0.f) ? m + logf(tot) : -INFINITY;
  }
  __syncthreads();
  // every rank's row of this (query, head) is read in groups of eight ranks,
  // all loads of a group in flight before the sums; a rank with no weight
  // (nothing selected there) adds nothing, whatever its row holds
  const int64_t rstride = static_cast<int64_t>(n_q) * H * dv;  // floats between ranks
  const float *src = outs + (static_cast<int64_t>(r) * H + h) * dv;
  float *dst = out + (static_cast<int64_t>(r) * H + h) * dv;
  const bool vec = (dv % 4) == 0 && (reinterpret_cast<uintptr_t>(outs) & 15u) == 0 &&
                   (reinterpret_cast<uintptr_t>(out) & 15u) == 0;
  if (vec) {
    for (int c = 4 * threadIdx.x; c < dv; c += 4 * blockDim.x) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int q0 = 0; q0 < R; q0 += 8) {
        float4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          v[u] = (q0 + u < R) ? __ldg(reinterpret_cast<const float4 *>(src + (q0 + u) * rstride + c))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float w = (q0 + u < R) ? wts[q0 + u] : 0.f;
          if (w != 0.f) {
            acc.x += w * v[u].x; acc.y += w * v[u].y; acc.z += w * v[u].z; acc.w += w * v[u].w;
          }
        }
      }
      *reinterpret_cast<float4 *>(dst + c) = acc;
    }
  } else {
    for (int c = threadIdx.x; c < dv; c += blockDim.x) {
      float acc = 0.f;
      for (int q0 = 0; q0 < R; q0 += 8) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = (q0 + u < R) ? __ldg(src + (q0 + u) * rstride + c) : 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float w = (q0 + u < R) ? wts[q0 + u] : 0.f;
          if (w != 0.f) acc += w * v[u];
        }
      }
      dst[c] = acc;
    }
  }
}

unsigned blocks_of(int64_t n, int per) { return static_cast<unsigned>((n + per - 1) / per); }

}  // namespace

dsa_status_t launch_cp_candidates(const float *scores, int64_t ld, int n_q, const int32_t *idx_local,
                                  int k, const int32_t *offsets, float *cand_s, int32_t *cand_i,
                                  cudaStream_t s) {
  if (launch_pdl(cp_candidates_kernel, dim3(blocks_of(static_cast<int64_t>(n_q) * k, 256)),
                 dim3(256), 0, s, 1, scores, ld, n_q, idx_local, k, offsets, cand_s,
                 cand_i) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

dsa_status_t launch_cp_pack(const float *all_s, int R, int n_q, int k, int64_t ld, float *packed,
                            int32_t *vlen, cudaStream_t s) {
  const int64_t n = std::max<int64_t>(static_cast<int64_t>(n_q) * R * k, n_q);
  if (launch_pdl(cp_pack_kernel, dim3(blocks_of(n, 256)), dim3(256), 0, s, 1, all_s, R, n_q, k,
                 ld, packed, vlen) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

dsa_status_t launch_cp_select(const int32_t *pos, const int32_t *all_i, int R, int n_q, int k,
                              const int32_t *my_off, const int32_t *my_len, int32_t *gidx,
                              int32_t *own, cudaStream_t s) {
  if (launch_pdl(cp_select_kernel, dim3(n_q), dim3(kSelThreads), 0, s, 1, pos, all_i, R, n_q, k,
                 my_off, my_len, gidx, own) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

dsa_status_t launch_cp_merge(const float *outs, const float *lses, int R, int n_q, int H, int dv,
                             float *out, float *lse, cudaStream_t s) {
  if (launch_pdl(cp_merge_kernel, dim3(n_q, H), dim3(128), 0, s, 1, outs, lses, R, n_q, H, dv,
                 out, lse) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

}  // namespace dsa
