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
// large for shared memory are re-read from global memory).  The exact k-th
// largest key T is found by radix select over the bits that vary in the row:
//   - the cluster-wide AND and OR of the keys (every CTA adds its own into all
//     CTAs' slots between the two halves of the first cluster barrier) fix
//     every bit that is the same in all keys (integer-valued scores leave long runs of those), so only
//     the span from the highest to the lowest varying bit is searched, in
//     11-bit digits (one to three passes);
//   - per pass, warps count their keys into shared-memory histograms shared
//     by a warp pair (the first digit spans the varying bits, so the keys
//     spread over many bins and the atomics rarely collide);
//   - the 2,048 bins form 16 coarse groups of 128, each owned by one CTA of
//     the cluster.  Each CTA folds its histograms, adds every non-zero bin
//     into the owner's merged histogram and its 16 coarse sums into every CTA
//     (red.shared::cluster.add: fire-and-forget, one remote add per bin);
//   - after one cluster barrier each CTA finds the coarse group holding the
//     k-th key from its own coarse sums, then reads that group's 128 fine bins
//     from the owner (one 16-byte remote load per lane of one warp).
// The kept set is {key > T} plus the first (k - #{key > T}) keys equal to T in
// index order.  Each warp walks a contiguous run of its CTA's segment in
// 32-key strips; per-warp and per-CTA counts of keys above / equal to T give
// every kept index its output position (the number of kept tokens with a
// lower index).  No sort, no global atomics, no global scratch.
#include <algorithm>

#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;                  // one 11-bit digit
constexpr int kDigitBits = 11;
constexpr int kCoarse = 16;                  // coarse groups of bins
constexpr int kCw = kBins / kCoarse;         // bins per coarse group (128)
constexpr int kPairs = kWarps / 2;           // histograms, one per warp pair
constexpr int kPrivWords = kPairs * kBins;
constexpr int kMaxPasses = 3;                // 32 bits in 11-bit digits
constexpr int kMergedWords = kMaxPasses * (kBins + kCoarse);
constexpr int kMaxC = 16;  // 16 needs the non-portable cluster size; 8 otherwise
// shared words before the key buffer: histograms, merged sets, warp AND/OR,
// warp counts, broadcast slots, pushed CTA counts, this CTA's AND/OR (+pad)
constexpr int kFixedWords =
    kPrivWords + kMergedWords + 2 * kWarps + 2 * kWarps + 4 + 2 * kMaxC + 4;

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

// the 11-bit digit of key u whose top bit is bit `top` (bits below bit 0 read as 0)
__device__ __forceinline__ uint32_t digit_of(uint32_t u, int shift) {
  return (shift >= 0 ? (u >> shift) : (u << -shift)) & (kBins - 1);
}
__device__ __forceinline__ uint32_t digit_mask(int shift) {
  return shift >= 0 ? (static_cast<uint32_t>(kBins - 1) << shift)
                    : (static_cast<uint32_t>(kBins - 1) >> -shift);
}
__device__ __forceinline__ uint32_t digit_bits(uint32_t d, int shift) {
  return shift >= 0 ? (d << shift) : (d >> -shift);
}

__global__ void __launch_bounds__(kThreads, 1) topk_kernel(const TopkParams p) {
  extern __shared__ __align__(16) uint32_t sm[];
  uint32_t *priv = sm;                                       // [kPairs][kBins]
  uint32_t *merged = priv + kPrivWords;                      // [kMaxPasses][kBins + kCoarse]
  uint32_t *wandor = merged + kMergedWords;                  // [2][kWarps] warp AND / OR
  int *wcnt = reinterpret_cast<int *>(wandor + 2 * kWarps);  // [2][kWarps] warp counts
  int *bcast = wcnt + 2 * kWarps;                            // [4]
  uint32_t *cnt_all = reinterpret_cast<uint32_t *>(bcast + 4);  // [kMaxC][2] pushed counts
  uint32_t *andor = cnt_all + 2 * kMaxC;  // [2] the row's ~AND / OR from every CTA, [2] pad
  uint64_t *bar = reinterpret_cast<uint64_t *>(andor + 4);
  uint32_t *keys = reinterpret_cast<uint32_t *>(bar + 2);    // [seg_cap], 16-byte aligned

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

  // zero the histograms and the AND / OR slots: the merged histograms and the
  // slots must be zero before any peer adds into them (first cluster arrive)
  {
    uint4 *z = reinterpret_cast<uint4 *>(priv);
    for (int i = tid; i < (kPrivWords + kMergedWords) / 4; i += kThreads)
      z[i] = make_uint4(0, 0, 0, 0);
    if (tid < 2) andor[tid] = 0u;
  }
  cluster_arrive();
  // keys into shared memory; AND / OR of this CTA's keys
  uint32_t k_and = 0xFFFFFFFFu, k_or = 0u;
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
      for (int i = tid; i < done; i += kThreads) {
        const uint32_t u = score_key(__uint_as_float(keys[i]));
        keys[i] = u;
        k_and &= u;
        k_or |= u;
      }
    }
    for (int i = done + tid; i < cnt; i += kThreads) {
      const uint32_t u = score_key(__ldg(src + i));
      keys[i] = u;
      k_and &= u;
      k_or |= u;
    }
  } else {
    for (int i = tid; i < cnt; i += kThreads) {
      const uint32_t u = score_key(srow[lo + i]);
      k_and &= u;
      k_or |= u;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    k_and &= __shfl_xor_sync(0xffffffffu, k_and, o);
    k_or |= __shfl_xor_sync(0xffffffffu, k_or, o);
  }
  if (lane == 0) { wandor[warp] = k_and; wandor[kWarps + warp] = k_or; }
  __syncthreads();
  cluster_wait();  // every CTA's slots are zero: add this CTA's AND / OR into all of them
  if (warp == 0) {
    uint32_t a = (lane < kWarps) ? wandor[lane] : 0xFFFFFFFFu;
    uint32_t o = (lane < kWarps) ? wandor[kWarps + lane] : 0u;
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) {
      a &= __shfl_xor_sync(0xffffffffu, a, s);
      o |= __shfl_xor_sync(0xffffffffu, o, s);
    }
    // slot 0 collects the OR of the complements (the complement of the AND)
    if (static_cast<uint32_t>(lane) < C) {
      red_dsmem_or_u32(map_to_rank(smem_u32(&andor[0]), lane), ~a);
      red_dsmem_or_u32(map_to_rank(smem_u32(&andor[1]), lane), o);
    }
  }
  cluster_sync();  // histograms zeroed everywhere, keys in place, the row's AND / OR local
  auto key_at = [&](int i) -> uint32_t { return cached ? keys[i] : score_key(srow[lo + i]); };
  const uint32_t g_and = ~andor[0];
  const uint32_t vary = g_and ^ andor[1];
  // bits that never vary are part of T already
  uint32_t pmask = ~vary, prefix = g_and & ~vary;
  const int hb = vary ? 31 - __clz(vary) : -1;
  const int lb = vary ? __ffs(vary) - 1 : 0;
  const int npass = vary ? (hb - lb + kDigitBits) / kDigitBits : 0;
  int krem = k;

  // contiguous run of this CTA's segment owned by warp w, in 32-key strips:
  // index order is (CTA, warp, strip, lane)
  const uint32_t lt_mask = (1u << lane) - 1u;
  const int run = ((cnt + kWarps * 32 - 1) / (kWarps * 32)) * 32;
  const int w_lo = min(cnt, warp * run), w_hi = min(cnt, w_lo + run);
  uint32_t *mine = priv + (warp >> 1) * kBins;
#pragma unroll 1
  for (int pass = 0; pass < npass; ++pass) {
    const int shift = hb - kDigitBits * pass - (kDigitBits - 1);  // may be negative
    uint32_t *mfine = merged + pass * (kBins + kCoarse);
    uint32_t *mcoarse = mfine + kBins;
    // histogram of the keys that match the prefix, four strips in flight
    for (int base = w_lo; base < w_hi; base += 128) {
      uint32_t bins[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = base + 32 * j + lane;
        uint32_t b = 0xFFFFFFFFu;  // no bin: past the run, or outside the prefix
        if (i < w_hi) {
          const uint32_t u = key_at(i);
          if ((u & pmask) == prefix) b = digit_of(u, shift);
        }
        bins[j] = b;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (bins[j] != 0xFFFFFFFFu) atomicAdd(&mine[bins[j]], 1u);
    }
    __syncthreads();
    // fold: thread t owns bins 4t .. 4t+3, clearing the pair histograms for
    // the next pass; each non-zero bin goes to its coarse group's owner, the
    // coarse sums (one group per warp) to every CTA
    {
      uint32_t v[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int h = 0; h < kPairs; ++h) {
        uint4 *ph = reinterpret_cast<uint4 *>(priv + h * kBins + 4 * tid);
        const uint4 x = *ph;
        v[0] += x.x; v[1] += x.y; v[2] += x.z; v[3] += x.w;
        *ph = make_uint4(0, 0, 0, 0);
      }
      const uint32_t owner = static_cast<uint32_t>(warp) % C;  // group = warp (kCw / 4 = 32)
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (v[q] != 0u) red_dsmem_add_u32(map_to_rank(smem_u32(&mfine[4 * tid + q]), owner), v[q]);
      uint32_t cs = v[0] + v[1] + v[2] + v[3];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) cs += __shfl_xor_sync(0xffffffffu, cs, o);
      if (lane == 0 && cs != 0u) {
        const uint32_t addr = smem_u32(&mcoarse[warp]);
        for (uint32_t r = 0; r < C; ++r) red_dsmem_add_u32(map_to_rank(addr, r), cs);
      }
    }
    cluster_sync();  // every CTA's counts are in the owners' and everyone's coarse sums
    if (warp == 0) {
      // coarse group holding the krem-th key from the top
      const uint32_t cc = (lane < kCoarse) ? mcoarse[lane] : 0u;
      int after = static_cast<int>(cc);  // inclusive suffix sum over lanes >= this one
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_down_sync(0xffffffffu, after, o);
        if (lane + o < 32) after += y;
      }
      after -= static_cast<int>(cc);  // keys in higher groups
      const bool hit = lane < kCoarse && after < krem && krem <= after + static_cast<int>(cc);
      const uint32_t hm = __ballot_sync(0xffffffffu, hit);
      const int gsel = hm ? __ffs(hm) - 1 : 0;  // exactly one group qualifies
      const int k1 = krem - __shfl_sync(0xffffffffu, after, gsel);
      // its 128 fine bins, four per lane, from the owner
      const uint32_t owner = static_cast<uint32_t>(gsel) % C;
      const uint32_t *fsrc = &mfine[gsel * kCw + 4 * lane];
      const uint4 f = (owner == c) ? *reinterpret_cast<const uint4 *>(fsrc)
                                   : ld_dsmem_v4(map_to_rank(smem_u32(fsrc), owner));
      const int tot = static_cast<int>(f.x + f.y + f.z + f.w);
      int above = tot;  // inclusive suffix sum, then keys in higher lanes' bins
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_down_sync(0xffffffffu, above, o);
        if (lane + o < 32) above += y;
      }
      above -= tot;
      const int fv[4] = {static_cast<int>(f.x), static_cast<int>(f.y), static_cast<int>(f.z),
                         static_cast<int>(f.w)};
#pragma unroll
      for (int q = 3; q >= 0; --q) {
        if (above < k1 && k1 <= above + fv[q]) {
          bcast[0] = gsel * kCw + 4 * lane + q;
          bcast[1] = k1 - above;
        }
        above += fv[q];
      }
    }
    __syncthreads();
    const uint32_t sel = static_cast<uint32_t>(bcast[0]);
    krem = bcast[1];
    prefix |= digit_bits(sel, shift);
    pmask |= digit_mask(shift);
    __syncthreads();  // bcast is rewritten by the next pass
  }
  const uint32_t T = prefix;  // the k-th largest key (every bit is fixed now)
  const int need_eq = krem;   // how many keys equal to T are kept

  // Ordered compaction: per-warp counts of keys above / equal to T, their
  // prefixes over warps and CTAs, then ballots place every kept key.
  {
    int gt = 0, eq = 0;
    for (int i = w_lo + lane; i < w_hi; i += 32) {
      const uint32_t u = key_at(i);
      gt += u > T;
      eq += u == T;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      gt += __shfl_xor_sync(0xffffffffu, gt, o);
      eq += __shfl_xor_sync(0xffffffffu, eq, o);
    }
    if (lane == 0) { wcnt[warp] = gt; wcnt[kWarps + warp] = eq; }
  }
  int *wgt = wcnt;  // [kWarps] per-warp counts, then exclusive prefixes
  int *weq = wcnt + kWarps;
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

// Short rows (at most 8 x 1,024 keys): one CTA of 1,024 threads per row with
// the keys in registers, thread t holding keys [E*t, E*t + E), so thread order
// is index order.  The same radix select over the varying bits and the same
// kept set and output order as the cluster kernel, with block barriers in
// place of cluster barriers and a block scan in place of the ordered walk.
constexpr int kSmallThreads = 1024;
constexpr int kSmallWarps = kSmallThreads / 32;
constexpr int kSmallCopies = 4;  // private histograms, one per eight warps
constexpr int kWarpsPerCopy = kSmallWarps / kSmallCopies;
// longer rows go to clusters: at 16K keys two CTAs beat one, at 8K one wins
constexpr int kSmallMaxLen = 8 * kSmallThreads;
constexpr size_t kSmallSmem = (static_cast<size_t>(kSmallCopies) * kBins + 2 * kSmallWarps + 4) * 4;

template <int E>
__global__ void __launch_bounds__(kSmallThreads, 1) topk_small_kernel(const TopkParams p) {
  extern __shared__ __align__(16) uint32_t sm[];
  uint32_t *hist = sm;                            // [kSmallCopies][kBins]
  uint32_t *wred = hist + kSmallCopies * kBins;   // [2][kSmallWarps] warp partials
  int *bc = reinterpret_cast<int *>(wred + 2 * kSmallWarps);  // [4] broadcast
  const int tid = threadIdx.x, warp = warp_id(), lane = lane_id();
  const int row = blockIdx.x;
  const int k = p.k;
  int32_t *out = p.idx + static_cast<int64_t>(row) * k;

  // zero the histograms while the kernel before this one finishes
  {
    uint4 *z = reinterpret_cast<uint4 *>(hist);
    for (int i = tid; i < kSmallCopies * kBins / 4; i += kSmallThreads) z[i] = make_uint4(0, 0, 0, 0);
  }
  griddep_wait();
  griddep_launch_dependents();

  int n = p.valid_len ? p.valid_len[row] : p.causal_base + row + 1;
  if (static_cast<int64_t>(n) > p.ld) n = static_cast<int>(p.ld);
  if (n < 0) n = 0;
  if (n <= k) {  // every token is kept: 0..n-1, then -1
    for (int i = tid; i < k; i += kSmallThreads) out[i] = (i < n) ? i : -1;
    return;
  }

  // this thread's keys: nv valid ones of E
  const float *srow = p.scores + static_cast<int64_t>(row) * p.ld;
  const int base = tid * E;
  const int nv = max(0, min(E, n - base));
  uint32_t key[E];
  if (nv == E && (reinterpret_cast<uintptr_t>(srow) & 15u) == 0) {
#pragma unroll
    for (int j = 0; j < E / 4; ++j) {
      const float4 v = __ldg(reinterpret_cast<const float4 *>(srow + base) + j);
      key[4 * j] = score_key(v.x);
      key[4 * j + 1] = score_key(v.y);
      key[4 * j + 2] = score_key(v.z);
      key[4 * j + 3] = score_key(v.w);
    }
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) key[e] = (e < nv) ? score_key(__ldg(srow + base + e)) : 0u;
  }
  // the row's AND and OR fix every bit that does not vary
  uint32_t k_and = 0xFFFFFFFFu, k_or = 0u;
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (e < nv) { k_and &= key[e]; k_or |= key[e]; }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    k_and &= __shfl_xor_sync(0xffffffffu, k_and, o);
    k_or |= __shfl_xor_sync(0xffffffffu, k_or, o);
  }
  if (lane == 0) { wred[warp] = k_and; wred[kSmallWarps + warp] = k_or; }
  __syncthreads();
  if (warp == 0) {
    uint32_t a = wred[lane], o = wred[kSmallWarps + lane];
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) {
      a &= __shfl_xor_sync(0xffffffffu, a, s);
      o |= __shfl_xor_sync(0xffffffffu, o, s);
    }
    if (lane == 0) { bc[2] = static_cast<int>(a); bc[3] = static_cast<int>(o); }
  }
  __syncthreads();
  const uint32_t g_and = static_cast<uint32_t>(bc[2]);
  const uint32_t vary = g_and ^ static_cast<uint32_t>(bc[3]);
  uint32_t pmask = ~vary, prefix = g_and & ~vary;
  const int hb = vary ? 31 - __clz(vary) : -1;
  const int lb = vary ? __ffs(vary) - 1 : 0;
  const int npass = vary ? (hb - lb + kDigitBits) / kDigitBits : 0;
  int krem = k;
  uint32_t *mine = hist + (warp / kWarpsPerCopy) * kBins;
#pragma unroll 1
  for (int pass = 0; pass < npass; ++pass) {
    const int shift = hb - kDigitBits * pass - (kDigitBits - 1);  // may be negative
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (e < nv && (key[e] & pmask) == prefix) atomicAdd(&mine[digit_of(key[e], shift)], 1u);
    __syncthreads();
    // thread t owns bins 2t, 2t+1: fold the copies (clearing them for the next pass)
    uint32_t c0 = 0u, c1 = 0u;
#pragma unroll
    for (int h = 0; h < kSmallCopies; ++h) {
      uint2 *ph = reinterpret_cast<uint2 *>(hist + h * kBins + 2 * tid);
      const uint2 x = *ph;
      c0 += x.x;
      c1 += x.y;
      *ph = make_uint2(0u, 0u);
    }
    // keys in the bins of higher threads: suffix sums within the warp, then over warps
    const int local = static_cast<int>(c0 + c1);
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_down_sync(0xffffffffu, incl, o);
      if (lane + o < 32) incl += y;
    }
    if (lane == 0) wred[warp] = static_cast<uint32_t>(incl);
    __syncthreads();
    int wv = static_cast<int>(wred[lane]);  // suffix over the warps above
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_down_sync(0xffffffffu, wv, o);
      if (lane + o < 32) wv += y;
    }
    const int wabove = __shfl_sync(0xffffffffu, wv, (warp + 1) & 31);
    const int above = (warp < kSmallWarps - 1 ? wabove : 0) + incl - local;
    // the bin holding the krem-th key from the top (bin 2t+1 ranks above 2t)
    if (above < krem && krem <= above + static_cast<int>(c1)) {
      bc[0] = 2 * tid + 1;
      bc[1] = krem - above;
    } else if (above + static_cast<int>(c1) < krem && krem <= above + local) {
      bc[0] = 2 * tid;
      bc[1] = krem - above - static_cast<int>(c1);
    }
    __syncthreads();
    const uint32_t sel = static_cast<uint32_t>(bc[0]);
    krem = bc[1];
    prefix |= digit_bits(sel, shift);
    pmask |= digit_mask(shift);
  }
  const uint32_t T = prefix;  // the k-th largest key
  const int need_eq = krem;   // how many keys equal to T are kept

  // ordered compaction: exclusive prefix over threads (index order) of the
  // keys above and equal to T, packed as gt | eq << 16 (each below 2^15)
  int gt = 0, eq = 0;
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (e < nv) { gt += key[e] > T; eq += key[e] == T; }
  const uint32_t v = static_cast<uint32_t>(gt) | (static_cast<uint32_t>(eq) << 16);
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  __syncthreads();  // wred and bc reads of the last pass are done
  if (lane == 31) wred[warp] = incl;
  __syncthreads();
  uint32_t wv = wred[lane];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, wv, o);
    if (lane >= o) wv += y;
  }
  const uint32_t wexcl = warp ? __shfl_sync(0xffffffffu, wv, warp - 1) : 0u;
  const uint32_t pre = wexcl + incl - v;
  int erank = static_cast<int>(pre >> 16);
  int pos = static_cast<int>(pre & 0xFFFFu) + min(erank, need_eq);
#pragma unroll
  for (int e = 0; e < E; ++e) {
    if (e < nv) {
      const uint32_t u = key[e];
      bool keep = u > T;
      if (u == T) keep = erank++ < need_eq;
      if (keep) {
        if (pos < k) out[pos] = base + e;
        ++pos;
      }
    }
  }
}

// Long rows (up to 16 CTAs x 16 x 1,024 keys): the cluster scheme above with
// 1,024 threads per CTA and the segment's keys in registers, thread t holding
// keys [E*t, E*t + E) of its CTA's segment, and a block scan for the ordered
// compaction.
constexpr int kRegMaxSeg = 16 * kSmallThreads;
constexpr size_t kRegSmem = (static_cast<size_t>(kSmallCopies) * kBins + kMergedWords +
                             2 * kSmallWarps + 4 + 2 * kMaxC + 4) * 4;

template <int E>
__global__ void __launch_bounds__(kSmallThreads, 1) topk_creg_kernel(const TopkParams p) {
  extern __shared__ __align__(16) uint32_t sm[];
  uint32_t *priv = sm;                                         // [kSmallCopies][kBins]
  uint32_t *merged = priv + kSmallCopies * kBins;              // [kMaxPasses][kBins + kCoarse]
  uint32_t *wred = merged + kMergedWords;                      // [2][kSmallWarps]
  int *bc = reinterpret_cast<int *>(wred + 2 * kSmallWarps);  // [4] broadcast
  uint32_t *cnt_all = reinterpret_cast<uint32_t *>(bc + 4);   // [kMaxC][2] pushed counts
  uint32_t *andor = cnt_all + 2 * kMaxC;  // [2] the row's ~AND / OR from every CTA, [2] pad

  const int tid = threadIdx.x, warp = warp_id(), lane = lane_id();
  const uint32_t C = cluster_nctarank();
  const uint32_t c = cluster_ctarank();
  const int row = blockIdx.x / C;
  const int k = p.k;
  int32_t *out = p.idx + static_cast<int64_t>(row) * k;

  // zero the histograms and the AND / OR slots before any peer adds into them
  // (first cluster arrive), while the kernel before this one finishes
  {
    uint4 *z = reinterpret_cast<uint4 *>(priv);
    for (int i = tid; i < (kSmallCopies * kBins + kMergedWords) / 4; i += kSmallThreads)
      z[i] = make_uint4(0, 0, 0, 0);
    if (tid < 2) andor[tid] = 0u;
  }
  cluster_arrive();
  griddep_wait();
  griddep_launch_dependents();

  int n = p.valid_len ? p.valid_len[row] : p.causal_base + row + 1;
  if (static_cast<int64_t>(n) > p.ld) n = static_cast<int>(p.ld);
  if (n < 0) n = 0;
  if (n <= k) {  // every token is kept: 0..n-1, then -1 (the whole cluster)
    for (int i = c * kSmallThreads + tid; i < k; i += C * kSmallThreads) out[i] = (i < n) ? i : -1;
    cluster_wait();
    return;
  }

  const float *srow = p.scores + static_cast<int64_t>(row) * p.ld;
  const int seg = ((n + C - 1) / C + 3) & ~3;
  const int lo = min(n, static_cast<int>(c) * seg);
  const int cnt = max(0, min(n, lo + seg) - lo);
  const int base = tid * E;
  const int nv = max(0, min(E, cnt - base));
  uint32_t key[E];
  if (nv == E && (reinterpret_cast<uintptr_t>(srow + lo + base) & 15u) == 0) {
#pragma unroll
    for (int j = 0; j < E / 4; ++j) {
      const float4 v = __ldg(reinterpret_cast<const float4 *>(srow + lo + base) + j);
      key[4 * j] = score_key(v.x);
      key[4 * j + 1] = score_key(v.y);
      key[4 * j + 2] = score_key(v.z);
      key[4 * j + 3] = score_key(v.w);
    }
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) key[e] = (e < nv) ? score_key(__ldg(srow + lo + base + e)) : 0u;
  }
  uint32_t k_and = 0xFFFFFFFFu, k_or = 0u;
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (e < nv) { k_and &= key[e]; k_or |= key[e]; }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    k_and &= __shfl_xor_sync(0xffffffffu, k_and, o);
    k_or |= __shfl_xor_sync(0xffffffffu, k_or, o);
  }
  if (lane == 0) { wred[warp] = k_and; wred[kSmallWarps + warp] = k_or; }
  __syncthreads();
  cluster_wait();  // every CTA's slots are zero: add this CTA's AND / OR into all of them
  if (warp == 0) {
    uint32_t a = wred[lane], o = wred[kSmallWarps + lane];
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) {
      a &= __shfl_xor_sync(0xffffffffu, a, s);
      o |= __shfl_xor_sync(0xffffffffu, o, s);
    }
    // slot 0 collects the OR of the complements (the complement of the AND)
    if (static_cast<uint32_t>(lane) < C) {
      red_dsmem_or_u32(map_to_rank(smem_u32(&andor[0]), lane), ~a);
      red_dsmem_or_u32(map_to_rank(smem_u32(&andor[1]), lane), o);
    }
  }
  cluster_sync();  // the row's AND / OR are local
  const uint32_t g_and = ~andor[0];
  const uint32_t vary = g_and ^ andor[1];
  uint32_t pmask = ~vary, prefix = g_and & ~vary;
  const int hb = vary ? 31 - __clz(vary) : -1;
  const int lb = vary ? __ffs(vary) - 1 : 0;
  const int npass = vary ? (hb - lb + kDigitBits) / kDigitBits : 0;
  int krem = k;
  uint32_t *mine = priv + (warp / kWarpsPerCopy) * kBins;
#pragma unroll 1
  for (int pass = 0; pass < npass; ++pass) {
    const int shift = hb - kDigitBits * pass - (kDigitBits - 1);  // may be negative
    uint32_t *mfine = merged + pass * (kBins + kCoarse);
    uint32_t *mcoarse = mfine + kBins;
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (e < nv && (key[e] & pmask) == prefix) atomicAdd(&mine[digit_of(key[e], shift)], 1u);
    __syncthreads();
    // fold: thread t owns bins 2t, 2t+1 (coarse group t / 64 = warp / 2),
    // clearing the copies for the next pass; non-zero bins go to the group's
    // owner, the warp's sum into every CTA's coarse sums
    {
      uint32_t c0 = 0u, c1 = 0u;
#pragma unroll
      for (int h = 0; h < kSmallCopies; ++h) {
        uint2 *ph = reinterpret_cast<uint2 *>(priv + h * kBins + 2 * tid);
        const uint2 x = *ph;
        c0 += x.x;
        c1 += x.y;
        *ph = make_uint2(0u, 0u);
      }
      const int g = warp >> 1;
      const uint32_t owner = static_cast<uint32_t>(g) % C;
      if (c0 != 0u) red_dsmem_add_u32(map_to_rank(smem_u32(&mfine[2 * tid]), owner), c0);
      if (c1 != 0u) red_dsmem_add_u32(map_to_rank(smem_u32(&mfine[2 * tid + 1]), owner), c1);
      uint32_t ws = c0 + c1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ws += __shfl_xor_sync(0xffffffffu, ws, o);
      if (lane == 0 && ws != 0u) {
        const uint32_t addr = smem_u32(&mcoarse[g]);
        for (uint32_t r = 0; r < C; ++r) red_dsmem_add_u32(map_to_rank(addr, r), ws);
      }
    }
    cluster_sync();  // every CTA's counts are in the owners' and everyone's coarse sums
    if (warp == 0) {
      // coarse group holding the krem-th key from the top
      const uint32_t cc = (lane < kCoarse) ? mcoarse[lane] : 0u;
      int after = static_cast<int>(cc);  // inclusive suffix sum over lanes >= this one
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_down_sync(0xffffffffu, after, o);
        if (lane + o < 32) after += y;
      }
      after -= static_cast<int>(cc);  // keys in higher groups
      const bool hit = lane < kCoarse && after < krem && krem <= after + static_cast<int>(cc);
      const uint32_t hm = __ballot_sync(0xffffffffu, hit);
      const int gsel = hm ? __ffs(hm) - 1 : 0;  // exactly one group qualifies
      const int k1 = krem - __shfl_sync(0xffffffffu, after, gsel);
      // its 128 fine bins, four per lane, from the owner
      const uint32_t owner = static_cast<uint32_t>(gsel) % C;
      const uint32_t *fsrc = &mfine[gsel * kCw + 4 * lane];
      const uint4 f = (owner == c) ? *reinterpret_cast<const uint4 *>(fsrc)
                                   : ld_dsmem_v4(map_to_rank(smem_u32(fsrc), owner));
      const int tot = static_cast<int>(f.x + f.y + f.z + f.w);
      int above = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_down_sync(0xffffffffu, above, o);
        if (lane + o < 32) above += y;
      }
      above -= tot;
      const int fv[4] = {static_cast<int>(f.x), static_cast<int>(f.y), static_cast<int>(f.z),
                         static_cast<int>(f.w)};
#pragma unroll
      for (int q = 3; q >= 0; --q) {
        if (above < k1 && k1 <= above + fv[q]) {
          bc[0] = gsel * kCw + 4 * lane + q;
          bc[1] = k1 - above;
        }
        above += fv[q];
      }
    }
    __syncthreads();
    const uint32_t sel = static_cast<uint32_t>(bc[0]);
    krem = bc[1];
    prefix |= digit_bits(sel, shift);
    pmask |= digit_mask(shift);
    __syncthreads();  // bc is rewritten by the next pass
  }
  const uint32_t T = prefix;  // the k-th largest key
  const int need_eq = krem;   // how many keys equal to T are kept

  // ordered compaction: block scan of gt | eq << 16 (each below 2^15 within a
  // CTA), CTA totals pushed to every CTA, then each thread places its keys
  int gt = 0, eq = 0;
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (e < nv) { gt += key[e] > T; eq += key[e] == T; }
  const uint32_t v = static_cast<uint32_t>(gt) | (static_cast<uint32_t>(eq) << 16);
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wred[warp] = incl;
  __syncthreads();
  uint32_t wv = wred[lane];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, wv, o);
    if (lane >= o) wv += y;
  }
  const uint32_t wexcl = warp ? __shfl_sync(0xffffffffu, wv, warp - 1) : 0u;
  const uint32_t total = __shfl_sync(0xffffffffu, wv, 31);
  const uint32_t pre = wexcl + incl - v;
  if (tid == 0) {
    for (uint32_t r = 0; r < C; ++r) {
      st_dsmem_u32(map_to_rank(smem_u32(&cnt_all[2 * c]), r), total & 0xFFFFu);
      st_dsmem_u32(map_to_rank(smem_u32(&cnt_all[2 * c + 1]), r), total >> 16);
    }
  }
  cluster_sync();  // counts of every CTA are local; no remote access follows
  int gt_before = 0, eq_before = 0;
  for (uint32_t r = 0; r < c; ++r) {
    gt_before += static_cast<int>(cnt_all[2 * r]);
    eq_before += static_cast<int>(cnt_all[2 * r + 1]);
  }
  int erank = eq_before + static_cast<int>(pre >> 16);
  int pos = gt_before + static_cast<int>(pre & 0xFFFFu) + min(erank, need_eq);
#pragma unroll
  for (int e = 0; e < E; ++e) {
    if (e < nv) {
      const uint32_t u = key[e];
      bool keep = u > T;
      if (u == T) keep = erank++ < need_eq;
      if (keep) {
        if (pos < k) out[pos] = lo + base + e;
        ++pos;
      }
    }
  }
}

}  // namespace

// Largest cluster the device co-schedules for this kernel and shared memory
// size: 16 where the non-portable size is available, else 8.  Queried once.
int max_cluster_of(void (*kern)(const TopkParams), int threads, size_t smem, int *cached) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 8;
  if (cached[dev] == 0) {
    int best = 8;
    if (func_attr_once(reinterpret_cast<const void *>(kern),
                       cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(16, 1, 1);
      cfg.blockDim = dim3(threads, 1, 1);
      cfg.dynamicSmemBytes = smem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 16;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n > 0) best = 16;
    }
    cudaGetLastError();  // clear a rejected query
    cached[dev] = best;
  }
  return cached[dev];
}
int max_topk_cluster(size_t smem) {
  static int cached[64];
  return max_cluster_of(topk_kernel, kThreads, smem, cached);
}

dsa_status_t launch_topk(const TopkLaunch &a, cudaStream_t stream) {
  // rounded up to a multiple of 4 like the rows' stride, so that every row's
  // segment (at most the stride) fits the per-thread key count chosen here
  const int max_len = static_cast<int>(
      std::min<int64_t>(INT32_MAX & ~3, (std::max<int64_t>(1, a.max_len) + 3) & ~int64_t{3}));
  const size_t max_smem = device_max_smem_optin();
  if (func_attr_once(reinterpret_cast<const void *>(topk_kernel),
                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                     static_cast<int>(max_smem)) != cudaSuccess)
    return DSA_ERR_CUDA;
  TopkParams p;
  p.scores = a.scores;
  p.ld = a.ld;
  p.n_q = a.n_q;
  p.valid_len = a.valid_len;
  p.causal_base = a.causal_base;
  p.k = a.k;
  p.idx = a.idx;
  p.seg_cap = 0;
  p.wait_ns = wait_limit_ns();
  p.status = a.status;
  if (max_len <= kSmallMaxLen) {
    // short rows: one CTA per row, keys in registers
    if (func_attr_once(reinterpret_cast<const void *>(topk_small_kernel<4>),
                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                       static_cast<int>(kSmallSmem)) != cudaSuccess ||
        func_attr_once(reinterpret_cast<const void *>(topk_small_kernel<8>),
                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                       static_cast<int>(kSmallSmem)) != cudaSuccess)
      return DSA_ERR_CUDA;
    void (*kern)(const TopkParams) =
        max_len <= 4 * kSmallThreads ? topk_small_kernel<4> : topk_small_kernel<8>;
    if (launch_pdl(kern, dim3(static_cast<unsigned>(a.n_q)), dim3(kSmallThreads), kSmallSmem, stream,
                   1u, p) != cudaSuccess)
      return DSA_ERR_CUDA;
    return DSA_OK;
  }
  // about 4K keys per CTA, at most one wave of CTAs
  int C = (max_len + 4095) / 4096;
  C = std::min(C, std::max(1, device_sm_count() / std::max(1, a.n_q)));
  {
    // segments of at most 16K keys: 1,024 threads per CTA, keys in registers
    static int reg_cached[64];
    for (const void *k : {reinterpret_cast<const void *>(topk_creg_kernel<4>),
                          reinterpret_cast<const void *>(topk_creg_kernel<8>),
                          reinterpret_cast<const void *>(topk_creg_kernel<16>)})
      if (func_attr_once(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(kRegSmem)) != cudaSuccess)
        return DSA_ERR_CUDA;
    const int Cr = std::max(1, std::min(C, max_cluster_of(topk_creg_kernel<16>, kSmallThreads,
                                                          kRegSmem, reg_cached)));
    const int seg_r = ((max_len + Cr - 1) / Cr + 3) & ~3;
    if (seg_r <= kRegMaxSeg) {
      if (Cr > 8) {
        for (const void *k : {reinterpret_cast<const void *>(topk_creg_kernel<4>),
                              reinterpret_cast<const void *>(topk_creg_kernel<8>),
                              reinterpret_cast<const void *>(topk_creg_kernel<16>)})
          if (func_attr_once(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
            return DSA_ERR_CUDA;
      }
      void (*kern)(const TopkParams) = seg_r <= 4 * kSmallThreads   ? topk_creg_kernel<4>
                                       : seg_r <= 8 * kSmallThreads ? topk_creg_kernel<8>
                                                                    : topk_creg_kernel<16>;
      if (launch_pdl(kern, dim3(static_cast<unsigned>(a.n_q) * Cr), dim3(kSmallThreads), kRegSmem,
                     stream, static_cast<unsigned>(Cr), p) != cudaSuccess)
        return DSA_ERR_CUDA;
      return DSA_OK;
    }
  }
  C = std::max(1, std::min(C, max_topk_cluster(max_smem)));
  const int seg = ((max_len + C - 1) / C + 3) & ~3;
  const size_t fixed = 4 * static_cast<size_t>(kFixedWords) + 16 + 64;
  const int cap_max = static_cast<int>((max_smem - fixed) / 4) & ~3;
  const int seg_cap = std::min(seg, cap_max);
  const size_t smem = fixed + 4 * static_cast<size_t>(seg_cap);
  p.seg_cap = seg_cap;
  if (launch_pdl(topk_kernel, dim3(static_cast<unsigned>(a.n_q) * C), dim3(kThreads), smem,
                 stream, static_cast<unsigned>(C), p) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

}  // namespace dsa
