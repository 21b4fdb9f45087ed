// Step 2 of the DSA step: exact top-k with the stable lower-index tie rule.
//
// ("GLM on an A100, in Vx", section "The model": each query keeps the 2,048
// highest-scoring tokens, all of them below 2,048; section "How do we know it
// is right?": ties resolve as a stable argsort of -scores does, i.e. the lower
// token index wins.)
//
// Design: one thread-block cluster of C CTAs per row.  Each CTA owns a
// contiguous segment of the row and keeps the order-preserving 32-bit keys of
// its scores in shared memory (re-reading global memory only when a segment
// is larger than shared memory).  Three radix passes (11 + 11 + 10 bits) find
// the exact k-th largest key T: every CTA builds a shared-memory histogram
// (warp-aggregated atomics), the cluster barrier publishes it, and every CTA
// sums all C histograms through distributed shared memory and runs the same
// deterministic suffix scan.  The kept set is {key > T} plus the first
// (k - #{key > T}) keys equal to T in index order, which a block-wide scan
// compacts in ascending index order: output position = number of kept tokens
// with a lower index.  No sort, no global atomics, no global scratch.
#include <algorithm>

#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;

struct TopkParams {
  const float *scores;
  int64_t ld;
  int n_q;
  const int32_t *valid_len;
  int causal_base;
  int k;
  int32_t *idx;
  int seg_cap;  // keys a CTA can keep in shared memory
  DevStatus *status;
};

// exclusive suffix sum (sum over threads with a higher id)
__device__ __forceinline__ int block_exclusive_suffix(int v, int *warp_sums) {
  const int lane = lane_id(), warp = warp_id();
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_down_sync(0xffffffffu, x, o);
    if (lane + o < 32) x += y;
  }
  if (lane == 0) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = (lane < kWarps) ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_down_sync(0xffffffffu, s, o);
      if (lane + o < 32) s += y;
    }
    if (lane < kWarps) warp_sums[lane] = s;
  }
  __syncthreads();
  const int after = (warp + 1 < kWarps) ? warp_sums[warp + 1] : 0;
  __syncthreads();
  return after + x - v;
}

__global__ void __launch_bounds__(kThreads, 1) topk_kernel(const TopkParams p) {
  extern __shared__ uint32_t sm[];
  uint32_t *hist = sm;                                         // [2][kBins]
  int *warp_sums = reinterpret_cast<int *>(sm + 2 * kBins);    // [2 * kWarps]
  int *bcast = warp_sums + 2 * kWarps;                         // [8]
  uint32_t *cnts = reinterpret_cast<uint32_t *>(bcast + 8);    // [2] per-CTA gt / eq counts
  uint32_t *keys = cnts + 8;                                   // [seg_cap]

  griddep_wait();
  griddep_launch_dependents();
  const uint32_t C = cluster_nctarank();
  const uint32_t c = cluster_ctarank();
  const int row = blockIdx.x / C;
  const int tid = threadIdx.x;
  const int k = p.k;
  int32_t *out = p.idx + static_cast<int64_t>(row) * k;

  int n = p.valid_len ? p.valid_len[row] : p.causal_base + row + 1;
  if (static_cast<int64_t>(n) > p.ld) n = static_cast<int>(p.ld);
  if (n < 0) n = 0;

  if (n <= k) {  // every token is kept: 0..n-1, then -1
    for (int i = c * kThreads + tid; i < k; i += C * kThreads) out[i] = (i < n) ? i : -1;
    return;  // the whole cluster takes this branch; no shared memory was shared
  }

  const float *srow = p.scores + static_cast<int64_t>(row) * p.ld;
  const int seg = ((n + C - 1) / C + 3) & ~3;
  const int lo = min(n, static_cast<int>(c) * seg);
  const int cnt = max(0, min(n, lo + seg) - lo);
  const bool cached = seg <= p.seg_cap;
  if (cached) {
    // every load of a batch in flight before the first is used
    const float *src = srow + lo;
    int done = 0;
    if ((reinterpret_cast<uintptr_t>(src) & 15u) == 0) {
      const int nv = cnt >> 2;
      const float4 *s4 = reinterpret_cast<const float4 *>(src);
      uint4 *k4 = reinterpret_cast<uint4 *>(keys);
      for (int base = 0; base < nv; base += kThreads * 8) {
        float4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int i = base + j * kThreads + tid;
          if (i < nv) v[j] = __ldg(s4 + i);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int i = base + j * kThreads + tid;
          if (i < nv)
            k4[i] = make_uint4(score_key(v[j].x), score_key(v[j].y), score_key(v[j].z),
                               score_key(v[j].w));
        }
      }
      done = nv << 2;
    }
    for (int i = done + tid; i < cnt; i += kThreads) keys[i] = score_key(__ldg(src + i));
  }
  __syncthreads();
  auto key_at = [&](int i) -> uint32_t { return cached ? keys[i] : score_key(srow[lo + i]); };

  uint32_t prefix = 0, pmask = 0;
  int krem = k;
  const int lane = lane_id();
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    // two histogram buffers: a peer may still read this pass's buffer while
    // this CTA fills the next one; the cluster barrier of the next pass
    // separates a buffer's reads from its reuse two passes later
    uint32_t *hb = hist + (pass & 1) * kBins;
    const int shift = (pass == 0) ? 21 : (pass == 1 ? 10 : 0);
    const uint32_t bmask = (pass < 2) ? 0x7FFu : 0x3FFu;
    for (int i = tid; i < kBins; i += kThreads) hb[i] = 0u;
    __syncthreads();
    for (int base = 0; base < cnt; base += kThreads) {
      const int i = base + tid;
      bool match = false;
      uint32_t bin = 0u;
      if (i < cnt) {
        const uint32_t u = key_at(i);
        match = (u & pmask) == prefix;
        bin = (u >> shift) & bmask;
      }
      // lanes with the same bin add once, with the count of the group
      const uint32_t mm = __ballot_sync(0xffffffffu, match);
      if (match) {
        const uint32_t peers = __match_any_sync(mm, bin);
        if (lane == __ffs(peers) - 1) atomicAdd(&hb[bin], __popc(peers));
      }
    }
    cluster_sync();  // every CTA's histogram of this pass is complete
    // global histogram: thread t owns bins 4t .. 4t+3; one 16-byte load per peer
    uint32_t gh[4] = {0u, 0u, 0u, 0u};
    {
      const uint32_t addr = smem_u32(&hb[4 * tid]);
      uint4 v[8];
#pragma unroll
      for (int r = 0; r < 8; ++r)
        if (r < static_cast<int>(C)) v[r] = ld_dsmem_v4(map_to_rank(addr, r));
#pragma unroll
      for (int r = 0; r < 8; ++r)
        if (r < static_cast<int>(C)) { gh[0] += v[r].x; gh[1] += v[r].y; gh[2] += v[r].z; gh[3] += v[r].w; }
    }
    const int mine = static_cast<int>(gh[0] + gh[1] + gh[2] + gh[3]);
    int above = block_exclusive_suffix(mine, warp_sums);
    // the bin where the running count from the top reaches krem
#pragma unroll
    for (int q = 3; q >= 0; --q) {
      const int h = static_cast<int>(gh[q]);
      if (above < krem && krem <= above + h) { bcast[0] = 4 * tid + q; bcast[1] = krem - above; }
      above += h;
    }
    __syncthreads();
    const uint32_t sel = static_cast<uint32_t>(bcast[0]);
    krem = bcast[1];
    prefix |= sel << shift;
    pmask |= bmask << shift;
  }
  const uint32_t T = prefix;   // the k-th largest key
  const int need_eq = krem;    // how many keys equal to T are kept

  // Ordered compaction.  Warp w owns the contiguous run [w*run, (w+1)*run) of
  // this CTA's segment and walks it in 32-key strips, so index order is
  // (CTA, warp, strip, lane).  Pass A counts keys above / equal to T per warp;
  // the CTA totals go to the cluster; pass B emits each kept index at
  // position = kept tokens with a lower index, found by ballots.
  const int warp = warp_id();
  const uint32_t lt_mask = (1u << lane) - 1u;
  const int run = ((cnt + kWarps * 32 - 1) / (kWarps * 32)) * 32;
  const int w_lo = min(cnt, warp * run), w_hi = min(cnt, w_lo + run);
  int gt_w = 0, eq_w = 0;
  for (int base = w_lo; base < w_hi; base += 32) {
    const int i = base + lane;
    const uint32_t u = (i < w_hi) ? key_at(i) : 0u;
    gt_w += __popc(__ballot_sync(0xffffffffu, i < w_hi && u > T));
    eq_w += __popc(__ballot_sync(0xffffffffu, i < w_hi && u == T));
  }
  int *wgt = warp_sums;        // [kWarps] per-warp counts, then exclusive prefixes
  int *weq = warp_sums + kWarps;
  if (lane == 0) { wgt[warp] = gt_w; weq[warp] = eq_w; }
  __syncthreads();
  if (tid == 0) {
    int g = 0, e = 0;
    for (int w = 0; w < kWarps; ++w) {
      const int a = wgt[w], b = weq[w];
      wgt[w] = g; weq[w] = e;
      g += a; e += b;
    }
    cnts[0] = static_cast<uint32_t>(g);
    cnts[1] = static_cast<uint32_t>(e);
  }
  cluster_sync();
  if (tid == 0) {
    uint32_t gt_before = 0, eq_before = 0;
    for (uint32_t r = 0; r < c; ++r) {
      gt_before += ld_dsmem_u32(map_to_rank(smem_u32(&cnts[0]), r));
      eq_before += ld_dsmem_u32(map_to_rank(smem_u32(&cnts[1]), r));
    }
    bcast[2] = static_cast<int>(gt_before);
    bcast[3] = static_cast<int>(eq_before);
  }
  __syncthreads();
  int erank = bcast[3] + weq[warp];                              // equal keys before this warp
  int pos = bcast[2] + wgt[warp] + min(erank, need_eq);          // kept keys before this warp
  for (int base = w_lo; base < w_hi; base += 32) {
    const int i = base + lane;
    const uint32_t u = (i < w_hi) ? key_at(i) : 0u;
    const bool gt = i < w_hi && u > T;
    const bool eq = i < w_hi && u == T;
    const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
    const bool keep = gt || (eq && erank + __popc(eqm & lt_mask) < need_eq);
    const uint32_t km = __ballot_sync(0xffffffffu, keep);
    if (keep) {
      const int o = pos + __popc(km & lt_mask);
      if (o < k) out[o] = lo + i;
    }
    pos += __popc(km);
    erank += __popc(eqm);
  }
  cluster_sync();  // keep this CTA's shared memory alive until peers are done
}

}  // namespace

dsa_status_t launch_topk(const TopkLaunch &a, cudaStream_t stream) {
  const int max_len = std::max(1, a.max_len);
  int C = (max_len + 4095) / 4096;
  C = std::max(1, std::min(C, 8));
  const int seg = ((max_len + C - 1) / C + 3) & ~3;
  const size_t fixed = 4 * (2 * kBins + 2 * kWarps + 8 + 8) + 64;
  const size_t max_smem = device_max_smem_optin();
  const int cap_max = static_cast<int>((max_smem - fixed) / 4);
  const int seg_cap = std::min(seg, cap_max);
  const size_t smem = fixed + 4 * static_cast<size_t>(seg_cap);

  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(max_smem)) != cudaSuccess)
      return DSA_ERR_CUDA;
    attr_set = true;
  }
  TopkParams p;
  p.scores = a.scores;
  p.ld = a.ld;
  p.n_q = a.n_q;
  p.valid_len = a.valid_len;
  p.causal_base = a.causal_base;
  p.k = a.k;
  p.idx = a.idx;
  p.seg_cap = seg_cap;
  p.status = a.status;

  if (launch_pdl(topk_kernel, dim3(static_cast<unsigned>(a.n_q) * C), dim3(kThreads), smem,
                 stream, static_cast<unsigned>(C), p) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

}  // namespace dsa
