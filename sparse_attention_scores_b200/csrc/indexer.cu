// Step 1 of the DSA step: indexer scores on tcgen05 tensor cores.
//
//   score[r, s] = sum_h w[r, h] * max(0, q_idx[r, h, :] . k_idx[s, :])
//
// ("GLM on an A100, in Vx", section "The model": a separate indexer scores
// every earlier token; section "How do we know it is right?": ReLU per
// indexer head before the heads are combined.)
//
// Design (sm_100a): persistent CTAs walk the work units, each first a
// contiguous share of most of them, then small chunks of the rest taken from a
// counter, so that the CTAs finish together.  A unit is one tile of 128 keys
// of one row group (decode: one sequence; causal prefill: G consecutive query
// rows, which share their keys).
// The key tile is the A operand (M = 128 keys, K = D_I), the queries of the
// group are the B operand (N = G * H_I), so one MMA chain per tile yields
// every (key, row, head) dot product in tensor memory.  Warp roles:
//   warp 0     TMA producer: 64-key pages straight from the paged cache
//              (two per tile) into a ring of shared-memory stages; the
//              query tile when the row group changes
//   warp 1     tcgen05.mma issuer (one thread), double-buffered accumulators
//   warps 2+   epilogue warpgroups taking alternate tiles: tcgen05.ld of a
//              128-lane accumulator, ReLU, head-weighted sum, coalesced fp32
//              stores; up to 8 accumulators let the MMA run ahead
//   last warp  (bf16 keys) an optional bulk copy that rides under the scan:
//              the host-buffer step's attention query, over the host link
// Decode runs two CTAs per SM (one epilogue warpgroup each) so that one CTA's
// pipeline bubbles are covered by the other; grouped prefill runs one CTA per
// SM with two epilogue warpgroups.
//
// FP8 index keys (K8): the cache holds each key as E4M3 bytes with one fp32
// scale per token ("GLM on an A100, in Vx", "INT4, FP8 and BF16": E4M3 bytes
// with a float32 scale per block; here a block is one token's key).  The byte
// pages go by TMA straight into the MMA's swizzled K-major layout and the
// tensor cores multiply them as E4M3 (kind::f8f6f4, half the bytes and half
// the MMA time of bf16 keys).  The bf16 queries enter as two E4M3 terms,
// q * 2^s = hi + lo with a power-of-two scale s per head (a small kernel
// before the indexer writes them, and folds 2^-s into the head weights); the
// two terms accumulate into one fp32 accumulator.  hi + lo holds all eight
// significant bits of a bf16 element unless the element is below about 2^-11
// of its head's largest one.  The epilogue multiplies a key's score by its
// scale, which commutes with the ReLU and the head sum because the scale is
// positive.
// Every wait is bounded in wall time; a time-out records an error in the
// status block, drains what is in flight, frees tensor memory and returns.
#include <algorithm>

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "dsa_internal.h"

namespace dsa {
namespace {

// producer warp, MMA warp, NEG epilogue warpgroups (NEG = 2: one CTA per SM;
// NEG = 1: two CTAs per SM, whose pipelines cover each other's bubbles), and
// for bf16 keys a copy warp (an optional bulk copy that runs under the scan)
template <int NEG, bool K8>
__host__ __device__ constexpr int threads_of() { return 64 + 128 * NEG + (K8 ? 0 : 32); }
constexpr int kMaxStages = 8;
constexpr int kMaxAcc = 8;         // accumulator buffers in tensor memory
constexpr int kTileKeys = 128;
constexpr int kBatch = 16;  // units whose pages the producer looks up at once (<= 16)
constexpr int kStaticPct = 50;  // share of the units split statically over the CTAs
constexpr int kDynChunk = 8;    // most units per counter chunk after that
constexpr int kDecodeStaticPct = 75;  // the same for decode (100: static only, one query buffer)
constexpr int kMinDynUnits = 8;       // units per CTA below which the split stays static
constexpr int kRing = 32;   // entries of the unit ring (> stages + accumulators + 2)

struct IndexerParams {
  const float *w;
  const int32_t *seq_lens;
  const int32_t *block_table;
  float *scores;
  int64_t ld;
  int n_q, H_I, D_I, causal, q_pos0;
  int max_pages, num_pages;
  int num_groups;
  int stages;
  int q_buffers;   // 1 or 2 query tiles in shared memory
  int static_pct;  // share of the units split statically, in percent
  int chunk;       // most units taken from the counter at a time (<= 16)
  uint64_t wait_ns;
  int debug_stall;  // the MMA issuer first waits on a barrier nothing arrives at
  const float *k_scale;  // K8: per physical key row [num_pages * 64]
  // [0] next unit to hand out, [1] CTAs finished (zero between launches: the
  // last CTA to finish resets both; the workspace init zeroes them first)
  int *work;
  DevStatus *status;
};

// bf16 keys: copy n16 16-byte words from src to dst under the scan (the
// host-buffer step's attention query, read from mapped host memory)
struct AuxCopy {
  const uint4 *src;
  uint4 *dst;
  int64_t n16;
};

// Tokens a row group must score (the longest row of the group).
template <int G>
__device__ __forceinline__ int group_keys(const IndexerParams &p, int g) {
  int n;
  if (!p.causal) {
    n = p.seq_lens[g];
  } else {
    const int last = min(g * G + G, p.n_q) - 1;
    n = p.q_pos0 + last + 1;
  }
  return max(0, min(min(n, p.max_pages * kPageSize), static_cast<int>(p.ld)));
}
// Tokens row r sees.
__device__ __forceinline__ int row_keys(const IndexerParams &p, int r) {
  const int n = p.causal ? p.q_pos0 + r + 1 : p.seq_lens[r];
  return max(0, min(min(n, p.max_pages * kPageSize), static_cast<int>(p.ld)));
}

// group containing unit u: the largest g with tile_start[g] <= u
__device__ __forceinline__ int locate(const int *tile_start, int ng, int u) {
  int lo = 0, hi = ng - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tile_start[mid] <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int G, int AW, int NEG, bool K8>
__global__ void __launch_bounds__(threads_of<NEG, K8>(), NEG == 1 ? 2 : 1)
    indexer_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                   const IndexerParams p, const __grid_constant__ AuxCopy aux) {
  constexpr int kThreads = threads_of<NEG, K8>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const int S = p.stages;
  const int nqb = p.q_buffers;
  constexpr int kEB = K8 ? 1 : 2;                // key / query bytes per element
  const int natoms = p.D_I * kEB / AW;          // swizzle atoms along K
  // K8: the tile's 128 key scales follow its key bytes (1 KB keeps stages aligned)
  const int kStageScales = kTileKeys * p.D_I * kEB;
  const int stage_bytes = kStageScales + (K8 ? 1024 : 0);
  const int ncols = G * p.H_I;                  // useful accumulator columns
  const int n_mma = (ncols + 15) & ~15;         // MMA N (multiple of 16)
  // K8: the hi and lo query terms, each [n_mma rows][D_I bytes], one after
  // the other; when both fit one MMA (N = 2 n_mma <= 256) they are its B
  // operand and the two products land side by side (hi, then lo columns)
  const int q_bytes = (K8 ? 2 : 1) * natoms * n_mma * AW;
  const bool fuse = K8 && 2 * n_mma <= 256;
  const uint32_t acc_stride = ((fuse ? 2 * n_mma : n_mma) + 31) & ~31;
  // as many accumulators as fit this CTA's share of the 512 columns (two CTAs
  // per SM: 256 each) (<= 8): the MMA warp runs that many tiles ahead of the
  // epilogue
  const int nacc = min(kMaxAcc, static_cast<int>((NEG == 1 ? 256u : 512u) / acc_stride));
  uint32_t tmem_cols = 32;
  while (tmem_cols < nacc * acc_stride) tmem_cols <<= 1;

  uint8_t *stage_base = smem;
  uint8_t *q_base = smem + S * stage_bytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(q_base + nqb * q_bytes);
  uint64_t *full = bars;                   // [S] key tile landed
  uint64_t *empty = bars + kMaxStages;     // [S] key tile consumed by the MMA
  uint64_t *qfull = bars + 2 * kMaxStages;
  uint64_t *qempty = qfull + 2;
  uint64_t *tfull = qempty + 2;
  uint64_t *tempty = tfull + kMaxAcc;
  uint64_t *drain = tempty + kMaxAcc;
  uint32_t *misc = reinterpret_cast<uint32_t *>(drain + 1);  // [0] tmem base, [1] abort
  int *scan_tmp = reinterpret_cast<int *>(misc + 4);          // [kThreads + 32]
  int *tile_start = scan_tmp + kThreads + 32;                 // [num_groups + 1]
  const int NG = p.num_groups;
  // (sequence number, unit, group) of this CTA's i-th unit, at [i % kRing]
  // (16-byte aligned: it is read and written as one vector)
  volatile int4 *uring = reinterpret_cast<volatile int4 *>(
      (reinterpret_cast<uintptr_t>(tile_start + NG + 1) + 15) & ~static_cast<uintptr_t>(15));

  const int warp = warp_id(), lane = lane_id();

  if (threadIdx.x == 0) {
    // K8: a stage is free once the MMA has run and the four epilogue warps that
    // take its unit have read their scales
    for (int i = 0; i < S; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], K8 ? 5 : 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&qfull[i], 1); mbar_init(&qempty[i], 1); }
    for (int i = 0; i < kMaxAcc; ++i) { mbar_init(&tfull[i], 1); mbar_init(&tempty[i], 4); }
    mbar_init(drain, 1);
    misc[1] = 0u;
    if (p.static_pct < 100 && nqb == 2)
      for (int i = 0; i < kRing; ++i) uring[i].x = -1;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) { tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmQ); }
  if (warp == 1) { tmem_alloc(&misc[0], tmem_cols); tmem_relinquish(); }

  // everything below may read what earlier work in the stream wrote
  griddep_wait();
  griddep_launch_dependents();
  // tile prefix over row groups (every CTA computes the same table)
  {
    const int per = (NG + kThreads - 1) / kThreads;
    const int g0 = min(NG, static_cast<int>(threadIdx.x) * per), g1 = min(NG, g0 + per);
    int local = 0;
    for (int g = g0; g < g1; ++g) local += (group_keys<G>(p, g) + kTileKeys - 1) / kTileKeys;
    // exclusive scan of `local` over the block: within warps by shuffles, then
    // over the warp totals (kThreads / 32 <= 32 of them) by the first warp
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) scan_tmp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int v = (lane < kThreads / 32) ? scan_tmp[lane] : 0;
      int wi = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += y;
      }
      if (lane < kThreads / 32) scan_tmp[kThreads + lane] = wi - v;  // warps before
      if (lane == kThreads / 32 - 1) tile_start[NG] = wi;
    }
    __syncthreads();
    int run = scan_tmp[kThreads + warp] + incl - local;
    for (int g = g0; g < g1; ++g) {
      tile_start[g] = run;
      run += (group_keys<G>(p, g) + kTileKeys - 1) / kTileKeys;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = misc[0];
  volatile uint32_t *abort_flag = &misc[1];

  const int total = tile_start[NG];
  // Work order: this CTA first walks its share of the first p.static_pct % of
  // the units (a contiguous range, so a row group's query tile is loaded once
  // per CTA), then takes chunks of at most p.chunk units from a counter shared by all
  // CTAs until none is left, so CTAs that run slower take fewer of them and
  // all finish together.  The MMA and epilogue warps know the static range;
  // the producer publishes each counter unit it issues (the i-th unit of the
  // CTA in uring[i % kRing]) and an end mark after the last.
  // (only with two query buffers, see the MMA issuer's group change, and
  // enough units per CTA for chunks to pay for the counter's latency; never
  // for FP8-key decode, whose kernel is then built without the counter paths)
  constexpr bool kMayDyn = NEG == 2 || !K8;
  const bool dyn = kMayDyn && p.static_pct < 100 && nqb == 2 &&
                   total >= kMinDynUnits * static_cast<int>(gridDim.x);
  const int st_total = static_cast<int>((static_cast<int64_t>(total) * min(p.static_pct, 100)) / 100);
  const int s0 = static_cast<int>((static_cast<int64_t>(st_total) * blockIdx.x) / gridDim.x);
  const int s1 = static_cast<int>((static_cast<int64_t>(st_total) * (blockIdx.x + 1)) / gridDim.x);
  // counter chunks: about two per CTA of what the static share leaves,
  // at most p.chunk units (the same value in every CTA)
  const int chunk = max(1, min(p.chunk, (total - st_total) / (2 * static_cast<int>(gridDim.x))));
  const uint32_t layout = (AW == 128) ? kLayoutSW128 : kLayoutSW64;
  // (lane 0) wait until uring holds the i-th entry; false on abort or time-out
  auto ring_get = [&](int i, int4 &e) -> bool {
    const uint32_t addr = smem_u32(const_cast<int4 *>(&uring[i % kRing]));
    const uint64_t t0 = global_timer_ns();
    uint32_t spins = 0;
    while (true) {
      asm volatile("ld.volatile.shared.v4.s32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(e.x), "=r"(e.y), "=r"(e.z), "=r"(e.w)
                   : "r"(addr)
                   : "memory");
      if (e.x == i) return true;
      if (++spins >= 16) {
        spins = 0;
        if (*abort_flag || global_timer_ns() - t0 > p.wait_ns) return false;
        __nanosleep(32);
      }
    }
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int stage = 0, qslot = 0, cur = -1;
    uint32_t phase = 0, qphase = 0;
    uint32_t armed = 0, armed_par = 0;  // stages with loads in flight, their phase parity
    bool ok = true;
    int seq = 0;  // units issued so far
    // batches of at most kBatch units: the static range, then counter chunks;
    // the counter is read one batch ahead so the atomic's latency is hidden
    int sb = s0;
    int pend = 0;           // lane 0: a counter value not yet used
    bool asked = false, dyn_done = false;
    auto ask = [&]() {
      if (lane == 0) pend = atomicAdd(p.work, chunk);
      asked = true;
    };
    auto take = [&](int &b_, int &n_) {
      b_ = total;
      n_ = 0;
      if (sb < s1) {
        b_ = sb;
        n_ = min(kBatch, s1 - sb);
        sb += n_;
        if (sb >= s1 && dyn && !asked) ask();
        return;
      }
      if (!dyn || dyn_done) return;
      if (!asked) ask();
      const int c = st_total + __shfl_sync(0xffffffffu, pend, 0);
      asked = false;
      if (c >= total) { dyn_done = true; return; }
      b_ = c;
      n_ = min(chunk, total - c);
      ask();
    };
    // lane-parallel page lookup: lane l resolves page (l & 1) of unit b_ + l/2;
    // the next batch is looked up while the current one is issued
    auto fetch = [&](int b_, int n_, int &g_, int &id_) {
      const int my_u = b_ + (lane >> 1);
      g_ = -1;
      id_ = -1;
      if ((lane >> 1) < n_) {
        g_ = locate(tile_start, NG, my_u);
        const int t = my_u - tile_start[g_];
        const int pg = 2 * t + (lane & 1);
        if (pg * kPageSize < group_keys<G>(p, g_)) {
          const int b = p.causal ? 0 : g_;
          const int id = p.block_table[static_cast<int64_t>(b) * p.max_pages + pg];
          if (id < 0 || id >= p.num_pages)
            report(p.status, kErrBadPage, (kKernIndexer << 24) | (pg & 0xFFFF));
          else
            id_ = id;
        }
      }
    };
    // (lane 0) the query tile of group gq into the next query buffer, once the
    // MMAs of the group that held it have completed
    uint32_t qarmed = 0, qarmed_par = 0;  // query buffers with loads in flight, their parity
    auto load_q = [&](int gq) -> bool {
      if (!mbar_wait(&qempty[qslot], qphase ^ 1u, p.wait_ns)) return false;
      mbar_arrive_expect_tx(&qfull[qslot], static_cast<uint32_t>((K8 ? 2 : 1) * natoms * ncols * AW));
      if (K8) {
        // hi plane rows [gq * ncols, ...), lo plane rows n_q * H_I further on
        uint8_t *qd = q_base + qslot * q_bytes;
        tma_load_2d(qd, &tmQ, 0, gq * ncols, &qfull[qslot]);
        tma_load_2d(qd + n_mma * AW, &tmQ, 0, p.n_q * p.H_I + gq * ncols, &qfull[qslot]);
      } else {
        for (int a = 0; a < natoms; ++a)
          tma_load_2d(q_base + qslot * q_bytes + a * n_mma * AW, &tmQ, a * (AW / 2), gq * ncols,
                      &qfull[qslot]);
      }
      qarmed |= 1u << qslot;
      qarmed_par = (qarmed_par & ~(1u << qslot)) | (qphase << qslot);
      if (++qslot == nqb) { qslot = 0; qphase ^= 1u; }
      return true;
    };
    int cb, cn, cur_g, cur_id;
    take(cb, cn);
    fetch(cb, cn, cur_g, cur_id);
    while (cn > 0 && ok) {
      int nb, nn, nxt_g, nxt_id;
      take(nb, nn);
      fetch(nb, nn, nxt_g, nxt_id);
      for (int i = 0; i < cn; ++i) {
        const int g = __shfl_sync(0xffffffffu, cur_g, 2 * i);
        const int id0 = __shfl_sync(0xffffffffu, cur_id, 2 * i);
        const int id1 = __shfl_sync(0xffffffffu, cur_id, 2 * i + 1);
        int okl = 1;
        if (lane == 0) {
          if (*abort_flag) okl = 0;
          if (okl && g != cur && !load_q(g)) okl = 0;
          if (okl && !mbar_wait(&empty[stage], phase ^ 1u, p.wait_ns)) okl = 0;
          if (okl && dyn) {
            // publish the unit before its stage is armed (the arrive releases it)
            asm volatile("st.volatile.shared.v4.s32 [%0], {%1, %2, %3, %4};" ::"r"(
                             smem_u32(const_cast<int4 *>(&uring[seq % kRing]))),
                         "r"(seq), "r"(cb + i), "r"(g), "r"(0)
                         : "memory");
          }
          if (okl) {
            // K8: each page also brings its 64 scales (256 bytes) into the stage
            const uint32_t page_bytes = kPageSize * p.D_I * kEB + (K8 ? kPageSize * 4 : 0);
            const uint32_t bytes = ((id0 >= 0) + (id1 >= 0)) * page_bytes;
            uint8_t *dst = stage_base + stage * stage_bytes;
            if (bytes == 0) {
              mbar_arrive(&full[stage]);
            } else {
              mbar_arrive_expect_tx(&full[stage], bytes);
              // an atom is AW bytes of a key row: AW / 2 bf16 or AW E4M3 elements
              for (int a = 0; a < natoms; ++a) {
                if (id0 >= 0)
                  tma_load_2d(dst + a * kTileKeys * AW, &tmK, a * (AW / kEB), id0 * kPageSize,
                              &full[stage]);
                if (id1 >= 0)
                  tma_load_2d(dst + a * kTileKeys * AW + kPageSize * AW, &tmK, a * (AW / kEB),
                              id1 * kPageSize, &full[stage]);
              }
              if (K8) {
                uint8_t *sc = dst + kStageScales;
                if (id0 >= 0)
                  bulk_load(sc, p.k_scale + static_cast<int64_t>(id0) * kPageSize, kPageSize * 4,
                            &full[stage]);
                if (id1 >= 0)
                  bulk_load(sc + kPageSize * 4, p.k_scale + static_cast<int64_t>(id1) * kPageSize,
                            kPageSize * 4, &full[stage]);
              }
              armed |= 1u << stage;
              armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
            }
          }
        }
        okl = __shfl_sync(0xffffffffu, okl, 0);
        if (!okl) { ok = false; break; }
        cur = g;
        ++seq;
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
      cb = nb;
      cn = nn;
      cur_g = nxt_g;
      cur_id = nxt_id;
    }
    if (lane == 0) {
      if (ok && dyn) {
        // end of the sequence, once for each epilogue warpgroup
        for (int k = 0; k < NEG; ++k)
          asm volatile("st.volatile.shared.v4.s32 [%0], {%1, %2, %3, %4};" ::"r"(
                           smem_u32(const_cast<int4 *>(&uring[(seq + k) % kRing]))),
                       "r"(seq + k), "r"(-1), "r"(-1), "r"(0)
                       : "memory");
      }
      if (dyn) {
        // this CTA reads the counter no more (the fence orders a request still
        // in flight after an abort); the last CTA to get here leaves both
        // counters at zero for the next launch, whose reads wait for this grid
        __threadfence();
        if (atomicAdd(&p.work[1], 1) == static_cast<int>(gridDim.x) - 1) {
          atomicExch(&p.work[0], 0);
          atomicExch(&p.work[1], 0);
        }
      }
      if (!ok && !*abort_flag) {
        *abort_flag = 1u;
        report(p.status, kErrTimeout, (kKernIndexer << 24) | 0x1);
      }
      for (int s = 0; s < S; ++s)  // drain loads in flight
        if (armed & (1u << s)) mbar_wait(&full[s], (armed_par >> s) & 1u, kDrainLimitNs);
      for (int s = 0; s < nqb; ++s)
        if (qarmed & (1u << s)) mbar_wait(&qfull[s], (qarmed_par >> s) & 1u, kDrainLimitNs);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = K8 ? idesc_e4m3_f32(kTileKeys, fuse ? 2 * n_mma : n_mma)
                                : idesc_bf16_f32(kTileKeys, n_mma, 0, 0);
      int stage = 0, qslot = 0, cur = -1, cur_slot = 0;
      uint32_t phase = 0, qphase = 0;
      bool ok = true;
      if (p.debug_stall && !mbar_wait(drain, 0, p.wait_ns)) ok = false;
      int gs = (s0 < s1) ? locate(tile_start, NG, s0) : 0;
      for (int i = 0; ok; ++i) {
        int g;
        if (i < s1 - s0) {
          while (tile_start[gs + 1] <= s0 + i) ++gs;
          g = gs;
        } else {
          if (!dyn) break;
          int4 e;
          if (!ring_get(i, e)) { ok = false; break; }
          if (e.y < 0) break;  // end of the sequence
          g = e.z;
        }
        if (g != cur) {
          // the previous group's query buffer is free once its MMAs complete.
          // (With the counter the MMA learns of a new group from the ring only
          // after the producer has loaded its query tile, so that load must not
          // wait for this commit: the grouped CTAs have a second query buffer.)
          if (cur >= 0) mma_commit(&qempty[cur_slot]);
          if (!mbar_wait(&qfull[qslot], qphase, p.wait_ns)) { ok = false; break; }
          cur = g;
          cur_slot = qslot;
          if (++qslot == nqb) { qslot = 0; qphase ^= 1u; }
        }
        // accumulator of the i-th unit of this CTA: i % nacc, its (i / nacc)-th use
        const int acc = i % nacc;
        const uint32_t aphase = static_cast<uint32_t>(i / nacc) & 1u;
        if (!mbar_wait(&full[stage], phase, p.wait_ns)) { ok = false; break; }
        if (!mbar_wait(&tempty[acc], aphase ^ 1u, p.wait_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem_base + acc * acc_stride;
        const uint32_t a_base = smem_u32(stage_base + stage * stage_bytes);
        const uint32_t b_base = smem_u32(q_base + cur_slot * q_bytes);
        if (K8 && fuse) {
          // E4M3 keys x [hi | lo] E4M3 query terms in one N = 2 n_mma operand
          // (one K atom: D_I = 128 bytes), 32 elements (32 bytes) per MMA
          for (int kk = 0; kk < AW / 32; ++kk)
            mma_e4m3(d, smem_desc(a_base + kk * 32, 16, 8 * AW, layout),
                     smem_desc(b_base + kk * 32, 16, 8 * AW, layout), idesc, kk != 0 ? 1u : 0u);
        } else if (K8) {
          // E4M3 keys x (hi + lo) E4M3 query terms, 32 elements (32 bytes) per MMA
          for (int term = 0; term < 2; ++term)
            for (int a = 0; a < natoms; ++a)
              for (int kk = 0; kk < AW / 32; ++kk) {
                const uint64_t adesc =
                    smem_desc(a_base + a * kTileKeys * AW + kk * 32, 16, 8 * AW, layout);
                const uint64_t bdesc = smem_desc(
                    b_base + term * natoms * n_mma * AW + a * n_mma * AW + kk * 32, 16, 8 * AW, layout);
                mma_e4m3(d, adesc, bdesc, idesc, (term | a | kk) != 0 ? 1u : 0u);
              }
        } else {
          for (int a = 0; a < natoms; ++a) {
            for (int kk = 0; kk < AW / 32; ++kk) {
              const uint64_t adesc = smem_desc(a_base + a * kTileKeys * AW + kk * 32, 16, 8 * AW, layout);
              const uint64_t bdesc = smem_desc(b_base + a * n_mma * AW + kk * 32, 16, 8 * AW, layout);
              mma_bf16(d, adesc, bdesc, idesc, (a | kk) != 0 ? 1u : 0u);
            }
          }
        }
        mma_commit(&empty[stage]);
        mma_commit(&tfull[acc]);
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
      if (!ok && !*abort_flag) {
        *abort_flag = 1u;
        report(p.status, kErrTimeout, (kKernIndexer << 24) | 0x2);
      }
      mma_commit(drain);  // every MMA issued above has completed once this fires
      mbar_wait(drain, 0, kDrainLimitNs);
    }
  } else if (K8 || warp < 2 + 4 * NEG) {
    // ------------------------------------------------------------ epilogue
    // (the FP8-key kernels have no copy warp, and are built without its code)
    // two warpgroups take alternate tiles; within a group, warp w reads the
    // tensor-memory lane quadrant w % 4 (keys 32*quad .. 32*quad+31 of the tile)
    const int quad = warp & 3;
    const int eg = (warp - 2) >> 2;
    const int key_in_tile = quad * 32 + lane;
    const int nchunks = (ncols + 31) / 32;
    const bool w_in_regs = (G == 1) && (p.H_I <= 32);
    float wreg[32];
    int wgroup = -1;
    bool ok = true;
    int gs = (s0 < s1) ? locate(tile_start, NG, s0) : 0;
    for (int i_unit = eg;; i_unit += NEG) {
      int u, g;
      if (i_unit < s1 - s0) {
        u = s0 + i_unit;
        while (tile_start[gs + 1] <= u) ++gs;
        g = gs;
      } else {
        if (!dyn) break;
        int4 e = make_int4(0, -1, -1, 0);
        int got = 1;
        if (lane == 0) got = ring_get(i_unit, e) ? 1 : 0;
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) { ok = false; break; }
        u = __shfl_sync(0xffffffffu, e.y, 0);
        g = __shfl_sync(0xffffffffu, e.z, 0);
        if (u < 0) break;  // end of the sequence
      }
      const int acc = i_unit % nacc;
      const uint32_t aphase = static_cast<uint32_t>(i_unit / nacc) & 1u;
      if (w_in_regs && g != wgroup) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          wreg[i] = (i < p.H_I) ? __ldg(p.w + static_cast<int64_t>(g) * p.H_I + i) : 0.f;
        wgroup = g;
      }
      // K8: this key's scale, which the producer copied into the unit's stage
      // with its key bytes; the stage is released once the MMA has run and
      // every epilogue warp has read its scales
      float kscale = 1.f;
      if (K8) {
        const int su = i_unit % S;
        const uint32_t sph = static_cast<uint32_t>(i_unit / S) & 1u;
        if (!__all_sync(0xffffffffu, mbar_wait(&full[su], sph, p.wait_ns))) { ok = false; break; }
        kscale = reinterpret_cast<const float *>(stage_base + su * stage_bytes + kStageScales)[key_in_tile];
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[su]);
      }
      if (__any_sync(0xffffffffu, *abort_flag != 0u)) { ok = false; break; }
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], aphase, p.wait_ns))) { ok = false; break; }
      tc_fence_after();
      float s[G];
#pragma unroll
      for (int j = 0; j < G; ++j) s[j] = 0.f;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * acc_stride;
      if (w_in_regs) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr, v);
        tmem_ld_wait();
        if (fuse) {
          // the lo term's products, n_mma columns on
          uint32_t v2[32];
          tmem_ld_32x32b_x32(taddr + n_mma, v2);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) + __uint_as_float(v2[i]));
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float x = __uint_as_float(v[i]);
          if (i < p.H_I) s[0] += wreg[i] * (x > 0.f ? x : 0.f);
        }
      } else {
        for (int c = 0; c < nchunks; ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(taddr + c * 32, v);
          // the 32 columns of a chunk belong to one row of the group (H_I is a
          // multiple of 32 when G > 1): row j, heads h0 .. h0 + nvalid - 1
          const int j = (G == 1) ? 0 : (c * 32) / p.H_I;
          const int h0 = c * 32 - j * p.H_I;
          const int nvalid = min(32, p.H_I - h0);
          const float *wrow = p.w + static_cast<int64_t>(min(g * G + j, p.n_q - 1)) * p.H_I + h0;
          tmem_ld_wait();
          if (fuse) {
            uint32_t v2[32];
            tmem_ld_32x32b_x32(taddr + n_mma + c * 32, v2);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) + __uint_as_float(v2[i]));
          }
          float part = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (i < nvalid) {
              const float x = __uint_as_float(v[i]);
              part += __ldg(wrow + i) * (x > 0.f ? x : 0.f);
            }
          }
          if (G == 1) {
            s[0] += part;
          } else {
#pragma unroll
            for (int jj = 0; jj < G; ++jj)
              if (jj == j) s[jj] += part;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      const int t = u - tile_start[g];
      const int key = t * kTileKeys + key_in_tile;
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const int r = p.causal ? g * G + j : g;
        if (r < p.n_q && key < row_keys(p, r))
          p.scores[static_cast<int64_t>(r) * p.ld + key] = K8 ? s[j] * kscale : s[j];
      }
    }
    if (!ok && lane == 0 && !*abort_flag) {
      *abort_flag = 1u;
      report(p.status, kErrTimeout, (kKernIndexer << 24) | 0x3);
    }
  } else {
    // ------------------------------------------------------------ copy warp
    // this CTA's share of the bulk copy, eight 16-byte loads in flight per
    // lane (the source may be host memory across the host link)
    if constexpr (!K8) {
      const int64_t n = aux.n16;
      const int64_t beg = (n * blockIdx.x) / gridDim.x, end = (n * (blockIdx.x + 1)) / gridDim.x;
      for (int64_t i0 = beg; i0 < end; i0 += 32 * 8) {
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int64_t i = i0 + u * 32 + lane;
          if (i < end) v[u] = aux.src[i];
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int64_t i = i0 + u * 32 + lane;
          if (i < end) aux.dst[i] = v[u];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

// The E4M3 query terms of the FP8-key indexer: per (row, head), the power-of-
// two scale 2^s that brings the largest |q| to at most 448 (the largest E4M3
// value), q * 2^s = hi + lo with hi = E4M3(q * 2^s) and lo = E4M3 of the
// remainder (both rounded to nearest even), and the head weight times 2^-s.
// One warp per (row, head); D_I / 32 elements per lane.
__global__ void __launch_bounds__(256) q8_prep_kernel(const uint16_t *q_idx, const float *w,
                                                       uint8_t *q8, float *w8, int n_q, int H_I,
                                                       int D_I) {
  griddep_wait();
  griddep_launch_dependents();
  const int wid = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (wid >= n_q * H_I) return;
  const int per = D_I / 32;  // 1, 2 or 4
  const uint16_t *src = q_idx + static_cast<int64_t>(wid) * D_I + lane * per;
  float v[4];
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[i] = (i < per) ? __uint_as_float(static_cast<uint32_t>(src[i]) << 16) : 0.f;
    m = fmaxf(m, fabsf(v[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  // m = f * 2^e, f in [0.5, 1): 2^s with s = 9 - e keeps m * 2^s = f * 512 <= 448
  // when f <= 0.875, else one power less
  int s = 0;
  if (m > 0.f) {
    int e;
    const float f = frexpf(m, &e);
    s = (f <= 0.875f) ? 9 - e : 8 - e;
  }
  uint32_t hi4 = 0u, lo4 = 0u;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (i >= per) break;
    const float x = ldexpf(v[i], s);
    const __nv_fp8_storage_t h = __nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
    const float hv = __half2float(__half(__nv_cvt_fp8_to_halfraw(h, __NV_E4M3)));
    const __nv_fp8_storage_t l = __nv_cvt_float_to_fp8(x - hv, __NV_SATFINITE, __NV_E4M3);
    hi4 |= static_cast<uint32_t>(h) << (8 * i);
    lo4 |= static_cast<uint32_t>(l) << (8 * i);
  }
  uint8_t *dh = q8 + static_cast<int64_t>(wid) * D_I + lane * per;
  uint8_t *dl = dh + static_cast<int64_t>(n_q) * H_I * D_I;
  for (int i = 0; i < per; ++i) {
    dh[i] = static_cast<uint8_t>(hi4 >> (8 * i));
    dl[i] = static_cast<uint8_t>(lo4 >> (8 * i));
  }
  if (lane == 0) w8[wid] = ldexpf(w[wid], -s);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
template <int G, int AW, int NEG, bool K8 = false>
dsa_status_t launch_impl(const IndexerLaunch &a, cudaStream_t stream) {
  constexpr int kThreads = threads_of<NEG, K8>();
  constexpr int kEB = K8 ? 1 : 2;
  const int natoms = a.D_I * kEB / AW;
  const int ncols = G * a.H_I;
  const int n_mma = (ncols + 15) & ~15;
  const int num_groups = a.causal ? (a.n_q + G - 1) / G : a.n_q;
  // the bulk copy rides on the bf16-key kernels' copy warp
  if (a.aux_bytes != 0 &&
      (K8 || a.aux_src == nullptr || a.aux_dst == nullptr || a.aux_bytes % 16 != 0 ||
       ((reinterpret_cast<uintptr_t>(a.aux_src) | reinterpret_cast<uintptr_t>(a.aux_dst)) & 15u) != 0))
    return DSA_ERR_INVALID_ARG;
  CUtensorMap tmK, tmQ;
  if (K8) {
    // byte keys [pages * 64 rows][D_I]; the query terms [2 * n_q * H_I rows][D_I]
    if (!make_map_2d_u8(&tmK, a.k8_pages, a.D_I, static_cast<uint64_t>(a.num_pages) * kPageSize,
                        AW, kPageSize, AW))
      return DSA_ERR_CUDA;
    if (!make_map_2d_u8(&tmQ, a.q8, a.D_I, 2ull * a.n_q * a.H_I, AW, ncols, AW))
      return DSA_ERR_CUDA;
  } else {
    if (!make_map_2d(&tmK, a.k_pages, a.D_I, static_cast<uint64_t>(a.num_pages) * kPageSize,
                     AW / 2, kPageSize, AW))
      return DSA_ERR_CUDA;
    if (!make_map_2d(&tmQ, a.q_idx, a.D_I, static_cast<uint64_t>(a.n_q) * a.H_I, AW / 2, ncols, AW))
      return DSA_ERR_CUDA;
  }
  (void)natoms;

  const int64_t max_keys = a.causal ? static_cast<int64_t>(a.q_pos0) + a.n_q : a.max_seq_len;
  const int64_t max_units = static_cast<int64_t>(num_groups) * ((max_keys + kTileKeys - 1) / kTileKeys);
  const int per_sm = (NEG == 1) ? 2 : 1;
  const int grid = static_cast<int>(
      std::max<int64_t>(1, std::min<int64_t>(static_cast<int64_t>(per_sm) * device_sm_count(), max_units)));
  const size_t stage_bytes = static_cast<size_t>(kTileKeys) * a.D_I * kEB + (K8 ? 1024 : 0);
  const size_t q_bytes = static_cast<size_t>(K8 ? 2 : 1) * natoms * n_mma * AW;
  // the counter needs a second query tile; bf16-key decode CTAs (two per SM
  // sharing its shared memory) take it, at the cost of a key stage (3 -> 2),
  // only when there can be enough units per CTA (the kernel checks the actual
  // count).  FP8-key decode CTAs stay static: their sixth stage was worth more
  // than the balance.
  const int pct = (NEG == 1) ? (K8 ? 100 : kDecodeStaticPct) : kStaticPct;
  const bool may_dyn = pct < 100 && max_units >= static_cast<int64_t>(kMinDynUnits) * grid;
  const int static_pct = may_dyn ? pct : 100;
  const int q_buffers = (NEG == 1 && !may_dyn) ? 1 : 2;
  const size_t fixed = 1024 /*align*/ + q_buffers * q_bytes +
                       8 * (2 * kMaxStages + 4 + 2 * kMaxAcc + 1) + 16 + 4 * (kThreads + 32) +
                       4 * ((num_groups + 4) & ~3) + (static_pct < 100 ? 16 + 16 * kRing : 0) + 64;
  const size_t max_smem = device_max_smem_optin();
  const size_t budget = std::min((NEG == 1) ? (device_smem_per_sm() / 2 - 1024) : max_smem, max_smem);
  if (budget <= fixed) return DSA_ERR_UNSUPPORTED;
  const int stages = static_cast<int>(std::min<size_t>(kMaxStages, (budget - fixed) / stage_bytes));
  if (stages < 2) return DSA_ERR_UNSUPPORTED;
  const size_t smem = fixed + stages * stage_bytes;

  if (func_attr_once(reinterpret_cast<const void *>(indexer_kernel<G, AW, NEG, K8>),
                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                     static_cast<int>(max_smem)) != cudaSuccess)
    return DSA_ERR_CUDA;

  IndexerParams p;
  p.w = a.w;
  p.seq_lens = a.seq_lens;
  p.block_table = a.block_table;
  p.scores = a.scores;
  p.ld = a.ld;
  p.n_q = a.n_q;
  p.H_I = a.H_I;
  p.D_I = a.D_I;
  p.causal = a.causal;
  p.q_pos0 = a.q_pos0;
  p.max_pages = a.max_pages;
  p.num_pages = a.num_pages;
  p.num_groups = num_groups;
  p.stages = stages;
  p.q_buffers = q_buffers;
  p.static_pct = static_pct;
  p.chunk = kDynChunk;
  p.wait_ns = wait_limit_ns();
  p.debug_stall = debug_stall() == kKernIndexer ? 1 : 0;
  p.k_scale = a.k_scale;
  p.status = a.status;
  p.work = reinterpret_cast<int *>(&a.status->pad[0]);
  AuxCopy aux;
  aux.src = static_cast<const uint4 *>(a.aux_src);
  aux.dst = static_cast<uint4 *>(a.aux_dst);
  aux.n16 = static_cast<int64_t>(a.aux_bytes / 16);
  if (launch_pdl(indexer_kernel<G, AW, NEG, K8>, dim3(grid), dim3(kThreads), smem, stream, 1, tmK, tmQ,
                 p, aux) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

}  // namespace

dsa_status_t launch_q8_prep(const uint16_t *q_idx, const float *w, uint8_t *q8, float *w8,
                            int n_q, int H_I, int D_I, cudaStream_t stream) {
  const unsigned grid = static_cast<unsigned>((static_cast<int64_t>(n_q) * H_I + 7) / 8);
  if (launch_pdl(q8_prep_kernel, dim3(grid), dim3(256), 0, stream, 1, q_idx, w, q8, w8, n_q, H_I,
                 D_I) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

dsa_status_t launch_indexer(const IndexerLaunch &a, cudaStream_t stream) {
  // causal prefill rows share keys: groups of 4 rows, one CTA per SM; decode
  // rows: one row per unit, two CTAs per SM
  const bool grouped = a.causal && (a.H_I % 32 == 0) && (4 * a.H_I <= 256);
  if (a.k8_pages != nullptr) {
    // E4M3 keys: 128-byte key rows (D_I = 128), the same CTA shapes as bf16
    if (a.D_I != 128) return DSA_ERR_UNSUPPORTED;
    return grouped ? launch_impl<4, 128, 2, true>(a, stream) : launch_impl<1, 128, 1, true>(a, stream);
  }
  if (a.D_I == 32) return grouped ? launch_impl<4, 64, 2>(a, stream) : launch_impl<1, 64, 1>(a, stream);
  return grouped ? launch_impl<4, 128, 2>(a, stream) : launch_impl<1, 128, 1>(a, stream);
}

}  // namespace dsa
