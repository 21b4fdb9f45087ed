// Step 2 of the DSA step: exact top-k with the stable lower-index tie rule.
//
// ("GLM on an A100, in Vx", section "The model": each query keeps the 2,048
// highest-scoring tokens, all of them below 2,048; section "How do we know it
// is right?": ties resolve as a stable argsort of -scores does, i.e. the lower
// token index wins.)
//
// Design: one thread-block cluster of C <= 16 CTAs per row.  Each CTA owns a
// contiguous segment of the row, pulls it into shared memory with one bulk
// copy and turns it into order-preserving 32-bit keys in place (segments too
// large for shared memory are re-read from global memory).  Three radix passes
// (11 + 11 + 10 bits) find the exact k-th largest key T:
//   - every warp counts its keys into a private shared-memory histogram
//     (no cross-warp contention, no match/vote aggregation);
//   - each CTA folds the 16 warp histograms and pushes its non-zero bins into
//     every CTA's merged histogram with remote reductions
//     (red.shared::cluster.add): fire-and-forget, no remote loads;
//   - after one cluster barrier every CTA scans the merged histogram itself.
// The kept set is {key > T} plus the first (k - #{key > T}) keys equal to T in
// index order.  Each warp walks a contiguous run of its CTA's segment in
// 32-key strips (the histogram passes walk the same order, so the last pass
// yields each warp's counts above / equal to T); per-CTA counts are pushed to
// every CTA; each kept index lands at position = number of kept tokens with a
// lower index.  No sort, no global atomics, no global scratch.
#include <algorithm>

#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;
constexpr int kMaxC = 16;  // 16 needs the non-portable cluster size; 8 otherwise

struct TopkParams {
  const float *scores;
  int64_t ld;
  int n_q;
  const int32_t *valid_len;
  int causal_base;
  int k;
  int32_t *idx;
  int seg_cap;  // keys a CTA can keep in shared memory
  uint64_t wait_ns;
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
  extern __shared__ __align__(16) uint32_t sm[];
  uint32_t *priv = sm;                                         // [kWarps][kBins]
  uint32_t *merged = priv + kWarps * kBins;                    // [2][kBins]
  int *warp_sums = reinterpret_cast<int *>(merged + 2 * kBins);  // [2 * kWarps]
  int *bcast = warp_sums + 2 * kWarps;                         // [4]
  uint32_t *cnt_all = reinterpret_cast<uint32_t *>(bcast + 4);   // [kMaxC][2] pushed counts
  uint64_t *bar = reinterpret_cast<uint64_t *>(cnt_all + 2 * kMaxC);
  uint32_t *keys = reinterpret_cast<uint32_t *>(bar + 2);      // [seg_cap], 16-byte aligned

  const int tid = threadIdx.x, warp = warp_id(), lane = lane_id();
  const uint32_t C = cluster_nctarank();
  const uint32_t c = cluster_ctarank();
  const int row = blockIdx.x / C;
  const int k = p.k;
  int32_t *out = p.idx + static_cast<int64_t>(row) * k;

  if (tid == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  griddep_wait();
  griddep_launch_dependents();

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

  // zero the histograms; merged[0] must be zero before any peer pushes into it
  {
    uint4 *z = reinterpret_cast<uint4 *>(priv);
    for (int i = tid; i < (kWarps + 2) * kBins / 4; i += kThreads) z[i] = make_uint4(0, 0, 0, 0);
  }
  if (cached && cnt > 0) {
    const float *src = srow + lo;
    int done = 0;
    if ((reinterpret_cast<uintptr_t>(src) & 15u) == 0 && cnt >= 4) {
      // one bulk copy of the first cnt & ~3 entries
      done = cnt & ~3;
      if (tid == 0) {
        mbar_arrive_expect_tx(bar, static_cast<uint32_t>(done) * 4u);
        bulk_load(keys, src, static_cast<uint32_t>(done) * 4u, bar);
        if (!mbar_wait(bar, 0u, p.wait_ns)) {
          report(p.status, kErrTimeout, (kKernTopk << 24) | 1u);
          mbar_wait(bar, 0u, kDrainLimitNs);  // let the copy land before the memory is reused
        }
      }
      __syncthreads();
      for (int i = tid; i < done; i += kThreads) keys[i] = score_key(__uint_as_float(keys[i]));
    }
    for (int i = done + tid; i < cnt; i += kThreads) keys[i] = score_key(__ldg(src + i));
  }
  cluster_sync();  // histograms zeroed everywhere, keys in place
  auto key_at = [&](int i) -> uint32_t { return cached ? keys[i] : score_key(srow[lo + i]); };

  uint32_t prefix = 0, pmask = 0;
  int krem = k;
  uint32_t *mine = priv + warp * kBins;
  // contiguous run of this CTA's segment owned by warp w, in 32-key strips:
  // index order is (CTA, warp, strip, lane)
  const uint32_t lt_mask = (1u << lane) - 1u;
  const int run = ((cnt + kWarps * 32 - 1) / (kWarps * 32)) * 32;
  const int w_lo = min(cnt, warp * run), w_hi = min(cnt, w_lo + run);
  int above_w = 0;  // keys of this lane above the 22-bit prefix (last pass)
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = (pass == 0) ? 21 : (pass == 1 ? 10 : 0);
    const uint32_t bmask = (pass < 2) ? 0x7FFu : 0x3FFu;
    uint32_t *mg = merged + (pass & 1) * kBins;
    // warp-private counts of the keys that still match the prefix; warp w
    // walks its contiguous run, so in the last pass its histogram (plus the
    // keys above the prefix) gives the warp's counts above / equal to T
    for (int base = w_lo; base < w_hi; base += 32) {
      const int i = base + lane;
      if (i < w_hi) {
        const uint32_t u = key_at(i);
        const uint32_t hi = u & pmask;
        if (hi == prefix) atomicAdd(&mine[(u >> shift) & bmask], 1u);
        else if (pass == 2 && hi > prefix) ++above_w;
      }
    }
    __syncthreads();
    // fold the warp histograms (thread t owns bins 4t .. 4t+3, clearing them
    // for the next pass) and push non-zero bins into every CTA's merged one
    {
      uint32_t v[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        uint4 *ph = reinterpret_cast<uint4 *>(priv + w * kBins + 4 * tid);
        const uint4 x = *ph;
        v[0] += x.x; v[1] += x.y; v[2] += x.z; v[3] += x.w;
        if (pass < 2) *ph = make_uint4(0, 0, 0, 0);  // the last pass's stay for the counts
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (v[q] == 0u) continue;
        const uint32_t addr = smem_u32(&mg[4 * tid + q]);
        for (uint32_t r = 0; r < C; ++r) red_dsmem_add_u32(map_to_rank(addr, r), v[q]);
      }
      // the other buffer is next pass's target: clear it before the barrier
      // (its last reader, the scan of the previous pass, is behind us)
      uint32_t *nx = merged + ((pass + 1) & 1) * kBins;
      *reinterpret_cast<uint4 *>(&nx[4 * tid]) = make_uint4(0, 0, 0, 0);
    }
    cluster_sync();  // every CTA's counts are in every merged histogram
    uint32_t gh[4];
    {
      const uint4 x = *reinterpret_cast<const uint4 *>(&mg[4 * tid]);
      gh[0] = x.x; gh[1] = x.y; gh[2] = x.z; gh[3] = x.w;
    }
    int above = block_exclusive_suffix(static_cast<int>(gh[0] + gh[1] + gh[2] + gh[3]), warp_sums);
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
    __syncthreads();  // bcast is rewritten by the next pass
  }
  const uint32_t T = prefix;   // the k-th largest key
  const int need_eq = krem;    // how many keys equal to T are kept

  // Ordered compaction.  Per-warp counts of keys above / equal to T: keys
  // above the 22-bit prefix, plus the last pass's warp histogram above /
  // at T's low 10 bits.
  const uint32_t b3 = T & 0x3FFu;
  int gt_w = above_w, eq_w = 0;
  for (uint32_t bin = b3 + 1 + lane; bin < 1024u; bin += 32) gt_w += static_cast<int>(mine[bin]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) gt_w += __shfl_xor_sync(0xffffffffu, gt_w, o);
  eq_w = static_cast<int>(mine[b3]);
  int *wgt = warp_sums;  // [kWarps] per-warp counts, then exclusive prefixes
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
    // push this CTA's totals into slot c of every CTA
    for (uint32_t r = 0; r < C; ++r) {
      st_dsmem_u32(map_to_rank(smem_u32(&cnt_all[2 * c]), r), static_cast<uint32_t>(g));
      st_dsmem_u32(map_to_rank(smem_u32(&cnt_all[2 * c + 1]), r), static_cast<uint32_t>(e));
    }
  }
  cluster_sync();  // counts of every CTA are local; no remote access follows
  int gt_before = 0, eq_before = 0;
  for (uint32_t r = 0; r < c; ++r) {
    gt_before += static_cast<int>(cnt_all[2 * r]);
    eq_before += static_cast<int>(cnt_all[2 * r + 1]);
  }
  int erank = eq_before + weq[warp];                       // equal keys before this warp
  int pos = gt_before + wgt[warp] + min(erank, need_eq);   // kept keys before this warp
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
}

}  // namespace

// Largest cluster the device co-schedules for this kernel and shared memory
// size: 16 where the non-portable size is available, else 8.  Queried once.
int max_topk_cluster(size_t smem) {
  static int cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 8;
  if (cached[dev] == 0) {
    int best = 8;
    if (cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
        cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(16, 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = smem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 16;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, topk_kernel, &cfg) == cudaSuccess && n > 0) best = 16;
    }
    cudaGetLastError();  // clear a rejected query
    cached[dev] = best;
  }
  return cached[dev];
}

dsa_status_t launch_topk(const TopkLaunch &a, cudaStream_t stream) {
  const int max_len = std::max(1, a.max_len);
  const size_t max_smem = device_max_smem_optin();
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(max_smem)) != cudaSuccess)
      return DSA_ERR_CUDA;
    attr_set = true;
  }
  // about 4K keys per CTA, at most one wave of CTAs
  int C = (max_len + 4095) / 4096;
  C = std::min(C, std::max(1, device_sm_count() / std::max(1, a.n_q)));
  C = std::max(1, std::min(C, max_topk_cluster(max_smem)));
  const int seg = ((max_len + C - 1) / C + 3) & ~3;
  const size_t fixed = 4 * ((kWarps + 2) * kBins + 2 * kWarps + 4 + 2 * kMaxC) + 16 + 64;
  const int cap_max = static_cast<int>((max_smem - fixed) / 4) & ~3;
  const int seg_cap = std::min(seg, cap_max);
  const size_t smem = fixed + 4 * static_cast<size_t>(seg_cap);
  TopkParams p;
  p.scores = a.scores;
  p.ld = a.ld;
  p.n_q = a.n_q;
  p.valid_len = a.valid_len;
  p.causal_base = a.causal_base;
  p.k = a.k;
  p.idx = a.idx;
  p.seg_cap = seg_cap;
  p.wait_ns = wait_limit_ns();
  p.status = a.status;
  if (launch_pdl(topk_kernel, dim3(static_cast<unsigned>(a.n_q) * C), dim3(kThreads), smem,
                 stream, static_cast<unsigned>(C), p) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

}  // namespace dsa
