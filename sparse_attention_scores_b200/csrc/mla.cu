// Step 3 of the DSA step: absorbed MLA attention over the selected latent rows.
//
//   z[h, j]   = scale * q[h, :] . L[idx_j, :]          (all R + P columns)
//   out[h, :] = sum_j softmax_j(z[h, :]) * L[idx_j, 0:R]   (V = the c_kv part)
//   lse[h]    = log sum_j exp(z[h, j])
//
// ("Self-contained GLM-5 serving stack: Just Vx kernels compiled to PTX",
// file list: absorbed MLA decode over compressed request-local KV, and the
// GPU-code paragraph: split online-softmax compressed MLA; "GLM on an A100,
// in Vx", "The model": one latent vector per token serves as key and value.)
//
// Design (sm_100a): a CTA of 8 warps owns one query row and a contiguous range
// of 128-key chunks of its selection (64-key chunks, the upper half of each
// tile masked, when few rows would leave SMs idle).  The 64-head absorbed query stays in
// shared memory for the whole range.  Per chunk:
//   gather   16-byte cp.async pieces of the selected latent rows straight
//            into a 128B-swizzled K-major tile (all threads, zero-fill for
//            unused slots)
//   S^T      tcgen05.mma, M = 128 keys, N = 64 heads, K = R + P, into TMEM
//   softmax  warp w reads keys 32*(w%4).. and heads 32*(w/4).. of S^T; per-head
//            max and sum over the 128 keys by a transposing butterfly of warp
//            shuffles; the running max moves only when it grows by more than
//            2^8, and then the TMEM accumulator is rescaled
//   O^T     += tcgen05.mma, M = 128 latent columns (R/128 blocks), N = 64
//            heads, K = 128 keys; the latent tile serves as V^T (MN-major view).
//            P = hi + lo (two bf16 terms, near-fp32 weights), written over the
//            rope atom, in two halves of 64 keys
// A row split over several CTAs writes its partial (m, l, O) to global
// scratch: O goes through shared memory one 128-column block at a time, and
// each block leaves with a bulk asynchronous store while the next is staged.
// A merge kernel, launched dependent on this one, combines the splits by
// log-sum-exp weights.
#include <algorithm>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kThreads = 256;         // 8 warps
constexpr int kChunk = 128;           // keys per chunk = MMA M
constexpr int kHeads = 64;            // head columns of every tile = MMA N
constexpr int kAtomL = kChunk * 128;  // bytes of one 64-column atom of the latent tile
constexpr int kAtomQ = kHeads * 128;  // bytes of one 64-column atom of the query tile
constexpr float kRescaleLog2 = 8.0f;
constexpr int kMaxMergeCluster = 8;  // splits merged inside one cluster
constexpr float kLn2 = 0.69314718055994531f;

enum : int { kMergeNone = 0, kMergeGlobal = 1 };

struct MlaParams {
  const uint16_t *q;
  const uint16_t *latent;  // paged latent rows [num_pages * 64][W]
  const uint8_t *latent8;  // E4M3 latent rows [num_pages * 64][W] (FP8 latent cache)
  const float *lat_scale;  // one fp32 scale per physical latent row (FP8 latent cache)
  const int32_t *idx;
  const int32_t *seq_lens;
  const int32_t *block_table;
  float *out;
  float *lse;
  float *part_o;   // [n_q, nsplit, R/128 blocks, 64 heads, 128]   (kMergeGlobal)
  float *part_ml;  // [n_q, nsplit, 2, 64]
  int n_q, H, R, W, topk, causal, q_pos0, max_pages, num_pages;
  int nsplit, chunks_per_split;
  int kc;   // selected keys per chunk: 128, or 64 when few rows leave SMs idle
  int ncb;  // CTAs per (row, split): 1, or one per 128-column block of the output
  int comb_ws;  // merge: warps per 128-column block (1, 2 or 4)
  int cluster_merge;  // the row's splits form one cluster and merge through DSMEM
  float scale_log2;
  uint64_t wait_ns;
  int debug_stall;  // wait once on a barrier nothing arrives at (tests the time-out path)
  int early_q;      // load the query tile before griddep_wait()
  DevStatus *status;
};

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Reduce 32 per-key values over the 32 keys (lanes) of a warp, for 32 heads at
// once: each butterfly step halves the heads a lane keeps and exchanges the
// other half with its partner; afterwards lane L holds head L's reduction.
// 31 shuffles instead of 32 x 5.
template <bool kMax, typename Get>
__device__ __forceinline__ float butterfly32(Get v) {
  const int lane = lane_id();
  auto op = [](float a, float b) { return kMax ? fmaxf(a, b) : a + b; };
  float a[16];
  {
    const bool up = lane & 16;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float lo_h = v(i), hi_h = v(i + 16);
      a[i] = op(up ? hi_h : lo_h, __shfl_xor_sync(0xffffffffu, up ? lo_h : hi_h, 16));
    }
  }
  float b[8];
  {
    const bool up = lane & 8;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      b[i] = op(up ? a[i + 8] : a[i], __shfl_xor_sync(0xffffffffu, up ? a[i] : a[i + 8], 8));
  }
  float c[4];
  {
    const bool up = lane & 4;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      c[i] = op(up ? b[i + 4] : b[i], __shfl_xor_sync(0xffffffffu, up ? b[i] : b[i + 4], 4));
  }
  float d[2];
  {
    const bool up = lane & 2;
#pragma unroll
    for (int i = 0; i < 2; ++i)
      d[i] = op(up ? c[i + 2] : c[i], __shfl_xor_sync(0xffffffffu, up ? c[i] : c[i + 2], 2));
  }
  const bool up = lane & 1;
  return op(up ? d[1] : d[0], __shfl_xor_sync(0xffffffffu, up ? d[0] : d[1], 1));
}

// The split merge of a row whose splits are the CTAs of one cluster (only the
// cluster instantiation of the kernel contains it).
// The row's splits are the CTAs of this cluster.  Each one sends its (m, l) to
// every CTA, then its O^T, scaled to the common maximum, in 32-column units
// (32 latent columns x 64 heads, 8 KB) to the unit's owner CTA (unit u =
// 4 mb + quadrant, owner u % C), into the owner's latent tile, which every CTA
// has finished with at the first barrier.  An owner sums its units over the C
// senders and writes the output.
__device__ __forceinline__ void cluster_merge_epilogue(const MlaParams &p, uint8_t *Ls, float *ml_all,
                                                    const float *mrun, const float *lrun,
                                                    float *alpha, float *red, uint32_t tmem_ol,
                                                    bool have_o, int row, int nmb) {
  const int tid = threadIdx.x, warp = warp_id(), lane = lane_id();
  const int q4 = warp & 3, hh = warp >> 2;
  const int R = p.R;
  const uint32_t C = cluster_nctarank(), me = cluster_ctarank();
  // every CTA of the cluster arrived (relaxed) at kernel entry: once this wait
  // returns, all of them have started and their shared memory may be written
  cluster_wait();
  if (tid < 2 * kHeads) {
    const int h = tid & (kHeads - 1);
    const float v = (tid < kHeads) ? mrun[h] : lrun[h];
    const uint32_t a = smem_u32(&ml_all[(me * 2 + (tid >> 6)) * kHeads + h]);
    for (uint32_t r = 0; r < C; ++r) st_dsmem_u32(map_to_rank(a, r), __float_as_uint(v));
  }
  cluster_sync();  // every split's loop is done and its (m, l) is everywhere
  if (tid < kHeads) {
    float M = -INFINITY;
    for (uint32_t r = 0; r < C; ++r) M = fmaxf(M, ml_all[(r * 2) * kHeads + tid]);
    float L = 0.f;
    for (uint32_t r = 0; r < C; ++r) {
      const float m = ml_all[(r * 2) * kHeads + tid];
      if (m != -INFINITY) L += exp2f(m - M) * ml_all[(r * 2 + 1) * kHeads + tid];
    }
    alpha[tid] = (mrun[tid] == -INFINITY) ? 0.f : exp2f(mrun[tid] - M);  // this split's weight
    red[tid] = (L > 0.f) ? 1.f / L : 0.f;
    if (me == 0 && tid < p.H)
      p.lse[static_cast<int64_t>(row) * p.H + tid] = (L > 0.f) ? (M + log2f(L)) * kLn2 : -INFINITY;
  }
  __syncthreads();
  const uint32_t recv = smem_u32(Ls);  // [units / C][C senders][32 columns][64 heads]
  for (int mb = 0; mb < nmb; ++mb) {
    uint32_t v[32];
    if (have_o) {
      tmem_ld_32x32b_x32(tmem_ol + mb * kHeads + 32 * hh, v);
      tmem_ld_wait();
    }
#pragma unroll
    for (int i = 0; i < 32; ++i)
      v[i] = have_o ? __float_as_uint(__uint_as_float(v[i]) * alpha[32 * hh + i]) : 0u;
    const uint32_t u = static_cast<uint32_t>(mb * 4 + q4);
    const uint32_t owner = u % C, slot = (u / C) * C + me;
    // column `lane`, heads 32 hh + 4 jj .. +3, at lane * 64 + (h ^ 4 (lane & 7))
    const uint32_t base = recv + (slot * 2048u + lane * 64u) * 4u;
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const uint32_t hsw = static_cast<uint32_t>((32 * hh + 4 * jj) ^ ((lane & 7) << 2));
      st_dsmem_v4(map_to_rank(base + hsw * 4u, owner), v[4 * jj], v[4 * jj + 1], v[4 * jj + 2],
                  v[4 * jj + 3]);
    }
  }
  cluster_sync();  // every unit is in its owner's buffer; no remote access follows
  const float *rbuf = reinterpret_cast<const float *>(Ls);
  const uint32_t nunits = static_cast<uint32_t>(nmb * 4);
  for (uint32_t j = 0; j * C + me < nunits; ++j) {
    const uint32_t u = j * C + me;
    const int col0 = static_cast<int>(u >> 2) * 128 + static_cast<int>(u & 3) * 32;
    const int c = lane;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int g = warp + 8 * k;  // heads 4g .. 4g+3
      const int hsw = (4 * g) ^ ((c & 7) << 2);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (uint32_t src = 0; src < C; ++src) {
        const float4 x =
            *reinterpret_cast<const float4 *>(rbuf + ((j * C + src) * 2048u + c * 64 + hsw));
        acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
      }
      const float a4[4] = {acc.x, acc.y, acc.z, acc.w};
      const int col = col0 + c;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int h = 4 * g + i;
        if (h < p.H && col < R)
          p.out[(static_cast<int64_t>(row) * p.H + h) * R + col] = a4[i] * red[h];
      }
    }
  }
}

// two E4M3 values (low byte first) as a bf16 pair, exactly: every E4M3 value
// is an f16 value and a bf16 value
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t v16) {
  uint32_t h;
  asm("{\n\t.reg .b16 a;\n\tcvt.u16.u32 a, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, a;\n\t}"
      : "=r"(h)
      : "r"(v16));
  const float lo = __half2float(__ushort_as_half(static_cast<unsigned short>(h & 0xFFFFu)));
  const float hi = __half2float(__ushort_as_half(static_cast<unsigned short>(h >> 16)));
  const __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&r);
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a));
  return v;
}
__device__ __forceinline__ void st_shared_v4(uint32_t a, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// Widen one 16-byte quarter (jq) of a latent row's E4M3 slices in place: the
// row's 64-byte slice of atom a sits in bytes [64, 128) of its 128-byte row of
// that atom (unswizzled); its 64 bf16 values go to the row's swizzled 16-byte
// units 2 jq and 2 jq + 1.  The four lanes holding a row's quarters must be
// in one warp, and every lane of the warp must call this together: all of
// them read before any of them writes.
__device__ __forceinline__ void widen_e4m3_quarter(uint32_t row_base, uint32_t sw, int jq, int nQ) {
  uint4 st[9];
#pragma unroll
  for (int a = 0; a < 9; ++a)
    if (a < nQ) st[a] = ld_shared_v4(row_base + a * kAtomL + 64 + 16 * jq);
  __syncwarp();
#pragma unroll
  for (int a = 0; a < 9; ++a) {
    if (a >= nQ) break;
    const uint32_t w4[4] = {st[a].x, st[a].y, st[a].z, st[a].w};
    uint32_t o[8];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      o[2 * t] = e4m3x2_to_bf16x2(w4[t] & 0xFFFFu);
      o[2 * t + 1] = e4m3x2_to_bf16x2(w4[t] >> 16);
    }
    st_shared_v4(row_base + a * kAtomL + (((2u * jq) ^ sw) << 4), make_uint4(o[0], o[1], o[2], o[3]));
    st_shared_v4(row_base + a * kAtomL + (((2u * jq + 1u) ^ sw) << 4), make_uint4(o[4], o[5], o[6], o[7]));
  }
  __syncwarp();
}

// kLat8: E4M3 latent rows with one fp32 scale per token, staged and widened
// in the tile as above; the token's scale multiplies its logit and its PV
// weight (the dequantized row is scale * e4m3(code)).
template <bool kClusterMerge, bool kLat8>
__global__ void __launch_bounds__(kThreads, 1) mla_kernel(const MlaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const int W = p.W;
  const int R = p.R;
  const int nQ = (W + 63) / 64;             // 64-column atoms of a latent/query row
  const int nmb = (R + 127) / 128;          // 128-row blocks of O^T
  const int nL = max(nQ, 2 * nmb);          // latent atoms allocated
  const bool p_overlays = nL > 2 * nmb;     // P reuses an atom that V never reads
  uint8_t *Ls = smem;
  uint8_t *Ps = p_overlays ? (Ls + (2 * nmb) * kAtomL) : (Ls + nL * kAtomL);
  uint8_t *Qs = Ls + nL * kAtomL + (p_overlays ? 0 : kAtomL);
  int *rowi = reinterpret_cast<int *>(Qs + nQ * kAtomQ);  // [128] physical row, -1 unused
  float *red = reinterpret_cast<float *>(rowi + kChunk);  // [4][64]
  float *mrun = red + 4 * kHeads;
  float *lrun = mrun + kHeads;
  float *alpha = lrun + kHeads;
  uint64_t *bar_s = reinterpret_cast<uint64_t *>(alpha + kHeads);
  uint64_t *bar_o = bar_s + 1;
  uint64_t *bar_drain = bar_o + 1;
  uint64_t *bar_stall = bar_drain + 1;
  // [0] tmem base, [1] rescale flag, [2] failed, [3] pad
  uint32_t *misc = reinterpret_cast<uint32_t *>(bar_stall + 1);
  // cluster merge: every split's (m, l) per head, [kMaxMergeCluster][2][64]
  float *ml_all = reinterpret_cast<float *>(misc + 4);
  float *kscale = ml_all + kMaxMergeCluster * 2 * kHeads;  // [128] per-key scale (kLat8)

  // the cluster merge writes into peers' shared memory: arrive now, wait
  // (for every peer to have started) just before the first remote store
  if constexpr (kClusterMerge) cluster_arrive_relaxed();
  const int tid = threadIdx.x, warp = warp_id(), lane = lane_id();
  const int q4 = warp & 3;   // tensor-memory lane quadrant: keys / rows 32*q4 ..
  const int hh = warp >> 2;  // head half: heads 32*hh ..
  const int split = blockIdx.x, row = blockIdx.y;
  // with few rows the 128-column blocks of the output go to separate CTAs
  // (each computes the chunk's logits and softmax, and its block of PV)
  const int mb0 = p.ncb > 1 ? static_cast<int>(blockIdx.z) : 0;
  const int nmb_l = p.ncb > 1 ? 1 : nmb;  // O^T blocks accumulated here
  const int b = p.causal ? 0 : row;
  const int kc = p.kc;
  const int nchunks = (p.topk + kc - 1) / kc;
  const int c_begin = split * p.chunks_per_split;
  const int c_end = min(nchunks, c_begin + p.chunks_per_split);
  const int cpr = W / 8;  // 16-byte pieces per query row

  uint32_t tmem_cols = 32;
  while (tmem_cols < static_cast<uint32_t>(kHeads + nmb_l * kHeads)) tmem_cols <<= 1;
  if (tid == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    mbar_init(bar_drain, 1);
    mbar_init(bar_stall, 1);
    misc[1] = 0u;
    misc[2] = 0u;
    fence_barrier_init();
  }
  if (tid < kHeads) { mrun[tid] = -INFINITY; lrun[tid] = 0.f; }
  if (warp == 0) { tmem_alloc(&misc[0], tmem_cols); tmem_relinquish(); }

  // earlier work in the stream may have written q, idx or the caches; in the
  // fused forward q predates the kernel before this one and loads first
  if (!p.early_q) griddep_wait();
  // the 64-head query tile (heads >= H zero-filled), 128B-swizzled, K-major
  {
    const uint16_t *qrow = p.q + static_cast<int64_t>(row) * p.H * W;
    const uint32_t qs = smem_u32(Qs);
    for (int h = warp; h < kHeads; h += kThreads / 32) {
      const bool ok = h < p.H;
      for (int cc = lane; cc < cpr; cc += 32) {
        const uint16_t *src = ok ? qrow + h * W + cc * 8 : p.q;
        cp_async_16(qs + (cc >> 3) * kAtomQ + h * 128 + (((cc & 7) ^ (h & 7)) << 4), src,
                    ok ? 16u : 0u);
      }
    }
    cp_async_commit();
  }
  // In the fused forward the block table predates this step too: stage the
  // row's page ids in the (still unused) latent tile, so the first chunk
  // resolves its rows without a second dependent global load.
  int staged_pages = 0;
  const int *tbl = reinterpret_cast<const int *>(Ls);
  if (p.early_q) {
    const int len = p.causal ? p.q_pos0 + row + 1 : p.seq_lens[b];
    const int npg = min(p.max_pages, (max(len, 0) + kPageSize - 1) / kPageSize);
    if (npg <= (nL * kAtomL) / 4) {
      staged_pages = npg;
      int *t = reinterpret_cast<int *>(Ls);
      for (int i = tid; i < npg; i += kThreads)
        t[i] = p.block_table[static_cast<int64_t>(b) * p.max_pages + i];
    }
    griddep_wait();
  }
  griddep_launch_dependents();
  const int limit = min(p.causal ? p.q_pos0 + row + 1 : p.seq_lens[b], p.max_pages * kPageSize);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_s = misc[0] + 32u * hh;                     // this warp's S^T columns
  const uint32_t tmem_o = misc[0] + kHeads;
  const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
  const uint32_t idesc_s = idesc_bf16_f32(kChunk, kHeads, 0, 0);
  const uint32_t idesc_pv = idesc_bf16_f32(kChunk, kHeads, 1, 1);
  uint32_t s_phase = 0, o_phase = 0;
  bool have_o = false;
  bool failed = false;

  if (p.debug_stall) {
    if (!mbar_wait(bar_stall, 0u, p.wait_ns)) misc[2] = 1u;
    __syncthreads();
    if (misc[2]) failed = true;
  }
  // Selected position of this thread's slot (threads 0..127) in the chunk
  // resolved next; the next chunk's position is loaded at the top of each
  // chunk and its page id before the PV product, so a chunk's rows resolve
  // without a dependent global load (the first chunk's come from the staged
  // table in the fused forward).
  auto slot_pos = [&](int ch) -> int {
    const int slot = ch * kc + tid;
    return (tid < kc && ch < c_end && slot < p.topk)
               ? p.idx[static_cast<int64_t>(row) * p.topk + slot]
               : -1;
  };
  int pos_n = slot_pos(c_begin);
  int page_n = -2;  // page id of pos_n when prefetched, -2 when not
  for (int ch = c_begin; ch < c_end && !failed; ++ch) {
    // resolve the 128 selected positions of this chunk to physical rows
    int valid = 0;
    if (tid < kChunk) {
      const int slot = ch * kc + tid;
      const int pos = pos_n;
      int phys = -1;
      if (pos >= 0) {
        if (pos >= limit) {
          report(p.status, kErrBadIndex, (kKernMla << 24) | (slot & 0xFFFF));
        } else {
          const int pg = pos / kPageSize;
          const int page = (page_n != -2) ? page_n
                           : (ch == c_begin && pg < staged_pages)
                               ? tbl[pg]
                               : p.block_table[static_cast<int64_t>(b) * p.max_pages + pg];
          if (page < 0 || page >= p.num_pages)
            report(p.status, kErrBadPage, (kKernMla << 24) | (slot & 0xFFFF));
          else
            phys = page * kPageSize + pos % kPageSize;
        }
      }
      rowi[tid] = phys;
      if constexpr (kLat8) kscale[tid] = (phys >= 0) ? p.lat_scale[phys] : 0.f;
      valid = phys >= 0;
      if (tid == 0) misc[1] = 0u;
    }
    pos_n = slot_pos(ch + 1);
    page_n = -2;
    if (__syncthreads_count(valid) == 0) continue;  // nothing to attend in this chunk
    // gather: the selected latent rows into the 128B-swizzled K-major tile,
    // 16 bytes per cp.async, eight threads per 128-byte atom row; unused rows
    // are zero-filled.  (TMA row gathers were measured to be issue-bound at
    // 15-19 GB/s per SM, whether the rows were in L2 or not; waiting and
    // issuing the logits product atom by atom was slower than one wait.)
    // Rows kc .. 127 of a 64-key chunk are never written: their keys are
    // masked and the PV product stops at key kc.
    if constexpr (kLat8) {
      // E4M3: quarter jq (16 bytes) of each row's 64-byte slice of atom a,
      // staged in the row's unswizzled 16-byte unit 4 + jq of that atom
      const uint32_t ls = smem_u32(Ls);
      for (int a = 0; a < nQ; ++a)
        for (int pc = tid; pc < kc * 4; pc += kThreads) {
          const int r = pc >> 2, jq = pc & 3;
          const int phys = rowi[r];
          const bool ok = phys >= 0 && a * 64 + 16 * jq < W;
          const uint8_t *src = ok ? p.latent8 + static_cast<int64_t>(phys) * W + a * 64 + 16 * jq
                                  : p.latent8;
          cp_async_16(ls + a * kAtomL + r * 128 + 64 + 16 * jq, src, ok ? 16u : 0u);
        }
      cp_async_commit();
      cp_async_wait_all();
      __syncthreads();  // every quarter of every row has landed
      // rows kc * 4 / kThreads at a time per warp, all lanes together
      for (int pc = tid; pc < kc * 4; pc += kThreads) {
        const int r = pc >> 2;
        widen_e4m3_quarter(smem_u32(Ls) + r * 128, static_cast<uint32_t>(r & 7), pc & 3, nQ);
      }
    } else {
      const uint32_t ls = smem_u32(Ls);
      const int per_atom = kc * 8;  // pieces of one atom: 8 per row
      for (int a = 0; a < nQ; ++a)
        for (int pc = tid; pc < per_atom; pc += kThreads) {
          const int r = pc >> 3, j = pc & 7, cc = a * 8 + j;
          const int phys = rowi[r];
          const bool ok = phys >= 0 && cc < cpr;
          const uint16_t *src = ok ? p.latent + static_cast<int64_t>(phys) * W + cc * 8 : p.latent;
          cp_async_16(ls + a * kAtomL + r * 128 + ((j ^ (r & 7)) << 4), src, ok ? 16u : 0u);
        }
      cp_async_commit();
    }
    cp_async_wait_all();  // this thread's pieces (and, first time round, the query tile)
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // S^T = L . Q^T  (M = 128 keys, N = 64 heads, K = W)
    if (tid == 0) {
      const uint32_t ls = smem_u32(Ls), qs = smem_u32(Qs);
      for (int a = 0; a < nQ; ++a)
        for (int kk = 0; kk < 4; ++kk) {
          if (a * 64 + kk * 16 >= W) break;
          mma_bf16(misc[0], smem_desc(ls + a * kAtomL + kk * 32, 16, 1024, kLayoutSW128),
                   smem_desc(qs + a * kAtomQ + kk * 32, 16, 1024, kLayoutSW128), idesc_s,
                   (a | kk) != 0 ? 1u : 0u);
        }
      mma_commit(bar_s);
    }
    if (!mbar_wait(bar_s, s_phase, p.wait_ns)) misc[2] = 1u;
    s_phase ^= 1u;
    tc_fence_after();
    __syncthreads();
    if (misc[2]) { failed = true; break; }

    // logits of key 32*q4 + lane for heads 32*hh .. 32*hh+31, log2 units
    const bool kvalid = rowi[q4 * 32 + lane] >= 0;
    // (E4M3 rows: the logit of the dequantized row, the key's scale applied)
    const float wk = kLat8 ? kscale[q4 * 32 + lane] : 1.f;
    float z[32];
    {
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem_s + lane_off, v);
      tmem_ld_wait();
      const float zs = p.scale_log2 * wk;
#pragma unroll
      for (int i = 0; i < 32; ++i) z[i] = kvalid ? __uint_as_float(v[i]) * zs : -INFINITY;
    }
    // per-head chunk max over the 128 keys
    red[q4 * kHeads + 32 * hh + lane] = butterfly32<true>([&](int i) { return z[i]; });
    __syncthreads();
    if (tid < kHeads) {
      const float mc = fmaxf(fmaxf(red[tid], red[kHeads + tid]),
                             fmaxf(red[2 * kHeads + tid], red[3 * kHeads + tid]));
      const float m_old = mrun[tid];
      const float m_new = (mc > m_old + kRescaleLog2) ? mc : m_old;
      const float a = (m_new == m_old) ? 1.f : exp2f(m_old - m_new);
      alpha[tid] = a;
      mrun[tid] = m_new;
      if (a != 1.f && have_o) misc[1] = 1u;
    }
    __syncthreads();
    // probabilities, split into a bf16 head and a bf16 tail: p = hi + lo to
    // about 2^-17, so the PV product keeps near-fp32 weights even when a few
    // keys dominate.  Sums use hi + lo.
    // (E4M3 rows: the PV weight is p times the key's scale; l sums p)
    uint32_t phi[16], plo[16];  // packed bf16 pairs of heads (2i, 2i+1) of this half
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int h = 32 * hh + 2 * i;
      float p0 = (z[2 * i] == -INFINITY) ? 0.f : exp2f(z[2 * i] - mrun[h]);
      float p1 = (z[2 * i + 1] == -INFINITY) ? 0.f : exp2f(z[2 * i + 1] - mrun[h + 1]);
      if constexpr (kLat8) {
        z[2 * i] = p0;
        z[2 * i + 1] = p1;
        p0 *= wk;
        p1 *= wk;
      }
      const __nv_bfloat162 hi = __floats2bfloat162_rn(p0, p1);
      const __nv_bfloat162 lo =
          __floats2bfloat162_rn(p0 - __low2float(hi), p1 - __high2float(hi));
      phi[i] = *reinterpret_cast<const uint32_t *>(&hi);
      plo[i] = *reinterpret_cast<const uint32_t *>(&lo);
    }
    {
      auto pf = [&](int i) {
        const uint32_t a = phi[i >> 1], c = plo[i >> 1];
        const uint32_t ha = (i & 1) ? (a & 0xFFFF0000u) : (a << 16);
        const uint32_t hc = (i & 1) ? (c & 0xFFFF0000u) : (c << 16);
        return __uint_as_float(ha) + __uint_as_float(hc);
      };
      if constexpr (kLat8)
        red[q4 * kHeads + 32 * hh + lane] = butterfly32<false>([&](int i) { return z[i]; });
      else
        red[q4 * kHeads + 32 * hh + lane] = butterfly32<false>(pf);
    }
    __syncthreads();
    if (tid < kHeads) {
      const float lc = (red[tid] + red[kHeads + tid]) + (red[2 * kHeads + tid] + red[3 * kHeads + tid]);
      lrun[tid] = lrun[tid] * alpha[tid] + lc;
    }
    // rescale the O accumulator when some head's running max moved
    if (misc[1]) {
      for (int mi = 0; mi < nmb_l; ++mi) {
        const uint32_t ta = tmem_o + lane_off + mi * kHeads + 32 * hh;
        uint32_t v[32];
        tmem_ld_32x32b_x32(ta, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i)
          v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha[32 * hh + i]);
        tmem_st_32x32b_x32(ta, v);
      }
      tmem_st_wait();
    }
    // the next chunk's page ids, from its positions loaded at the top
    if (tid < kChunk && pos_n >= 0 && pos_n < limit)
      page_n = p.block_table[static_cast<int64_t>(b) * p.max_pages + pos_n / kPageSize];
    // O^T += L^T . P^T  (M = 128 latent columns per block, N = 64 heads), in two
    // halves of 64 keys; each half multiplies by the hi and by the lo terms.
    // The 16 KB P region holds [hi | lo] for the 64 keys of one half.
    bool pv_failed = false;
    for (int half = 0; half < kc / 64; ++half) {
      if ((q4 >> 1) == half) {
        const int rk = 32 * (q4 & 1) + lane;
        const uint32_t base = smem_u32(Ps) + rk * 128;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t off = (((4 * hh + j) ^ (rk & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(base + off),
                       "r"(phi[4 * j]), "r"(phi[4 * j + 1]), "r"(phi[4 * j + 2]), "r"(phi[4 * j + 3])
                       : "memory");
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(base + 8192 + off),
                       "r"(plo[4 * j]), "r"(plo[4 * j + 1]), "r"(plo[4 * j + 2]), "r"(plo[4 * j + 3])
                       : "memory");
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      if (tid == 0) {
        const uint32_t ls = smem_u32(Ls), ps = smem_u32(Ps);
        for (int mi = 0; mi < nmb_l; ++mi)
          for (int part = 0; part < 2; ++part)
            for (int ks = 0; ks < 4; ++ks)
              mma_bf16(tmem_o + mi * kHeads,
                       smem_desc(ls + 2 * (mb0 + mi) * kAtomL + (half * 4 + ks) * 2048, kAtomL, 1024,
                                 kLayoutSW128),
                       smem_desc(ps + part * 8192 + ks * 2048, kAtomQ, 1024, kLayoutSW128),
                       idesc_pv, (have_o || half || part || ks) ? 1u : 0u);
        mma_commit(bar_o);
      }
      if (!mbar_wait(bar_o, o_phase, p.wait_ns)) misc[2] = 1u;
      o_phase ^= 1u;
      tc_fence_after();
      __syncthreads();
      if (misc[2]) { pv_failed = true; break; }
    }
    if (pv_failed) failed = true;
    have_o = true;
  }
  cp_async_wait_all();

  if (failed) {
    if (tid == 0) {
      report(p.status, kErrTimeout, (kKernMla << 24) | 1u);
      mma_commit(bar_drain);  // fires once every MMA issued above has completed
      mbar_wait(bar_drain, 0u, kDrainLimitNs);
    }
    if (tid < kHeads) { mrun[tid] = -INFINITY; lrun[tid] = 0.f; }
    have_o = false;
    __syncthreads();
  }

  if constexpr (kClusterMerge) {
    cluster_merge_epilogue(p, Ls, ml_all, mrun, lrun, alpha, red, tmem_o + lane_off, have_o, row,
                           nmb);
  } else if (p.nsplit == 1) {
    // the whole selection ran here: normalise and write the output
    for (int mi = 0; mi < nmb_l; ++mi) {
      uint32_t v[32];
      if (have_o) {
        tmem_ld_32x32b_x32(tmem_o + lane_off + mi * kHeads + 32 * hh, v);
        tmem_ld_wait();
      }
      const int r = (mb0 + mi) * 128 + q4 * 32 + lane;
      if (r < R) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int h = 32 * hh + i;
          if (h >= p.H) break;
          const float l = lrun[h];
          const float o = (have_o && l > 0.f) ? __uint_as_float(v[i]) / l : 0.f;
          p.out[(static_cast<int64_t>(row) * p.H + h) * R + r] = o;
        }
      }
    }
    if (tid < p.H && mb0 == 0) {
      const float l = lrun[tid];
      p.lse[static_cast<int64_t>(row) * p.H + tid] =
          (l > 0.f) ? (mrun[tid] + log2f(l)) * kLn2 : -INFINITY;
    }
  } else {
    // partial (m, l, O) of this split.  O^T leaves one 128-column block at a
    // time: staged as fp32 [64 heads][128] in shared memory (the latent tile
    // is free now), then written by a bulk asynchronous store that runs while
    // the next block is staged.
    float *Obuf = reinterpret_cast<float *>(Ls);
    float *dst = p.part_o + (static_cast<int64_t>(row) * p.nsplit + split) * nmb * kHeads * 128;
    if (tid < kHeads && mb0 == 0) {
      float *ml = p.part_ml + (static_cast<int64_t>(row) * p.nsplit + split) * 2 * kHeads;
      ml[tid] = mrun[tid];
      ml[kHeads + tid] = lrun[tid];
    }
    for (int mi = 0; mi < nmb_l; ++mi) {
      uint32_t v[32];
      if (have_o) {
        tmem_ld_32x32b_x32(tmem_o + lane_off + mi * kHeads + 32 * hh, v);
        tmem_ld_wait();
      }
      float *blk = Obuf + mi * kHeads * 128;
      const int cc = q4 * 32 + lane;
#pragma unroll
      for (int i = 0; i < 32; ++i) blk[(32 * hh + i) * 128 + cc] = have_o ? __uint_as_float(v[i]) : 0.f;
      fence_proxy_async_smem();
      __syncthreads();
      if (tid == 0) {
        asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                         reinterpret_cast<uint64_t>(dst + (mb0 + mi) * kHeads * 128)),
                     "r"(smem_u32(blk)), "r"(static_cast<uint32_t>(kHeads * 128 * 4))
                     : "memory");
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      }
    }
    if (tid == 0) {
      // the shared memory must stay valid until the stores have read it
      asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    __syncwarp();
    tmem_dealloc(misc[0], tmem_cols);
  }
}

// Merge the split partials of (row, head) over 128-column blocks:
//   out = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s,  lse = (M + log2 L) ln 2.
// Four warps per CTA: ws = p.comb_ws warps share one column block (warp
// taking every ws-th split) and the CTA covers 4 / ws blocks, so few splits
// give fat CTAs and many splits give short load chains.  Each lane owns four
// consecutive columns.  A warp issues the 16-byte loads of all its splits (at
// most 16) before it computes the merge weights, while its lanes load every
// split's (m, l) (nsplit <= 64), so it waits on memory once; the partial sums
// of a block's warps meet in shared memory.
constexpr int kCombineWarps = 4;
__global__ void __launch_bounds__(32 * kCombineWarps) combine_kernel(const MlaParams p) {
  constexpr int kBatch = 16;
  __shared__ float4 part[kCombineWarps][32];
  const int row = blockIdx.x, h = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ws = p.comb_ws, sub = warp % ws;
  const int mb = blockIdx.z * (kCombineWarps / ws) + warp / ws;
  const int nmb = (p.R + 127) / 128;
  griddep_wait();
  griddep_launch_dependents();
  const bool active = mb < nmb;  // warp-uniform
  const int c = 4 * lane;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (active) {
    const int64_t sstride = static_cast<int64_t>(nmb) * kHeads * 128;  // floats per split
    const float *po =
        p.part_o + (static_cast<int64_t>(row) * p.nsplit * nmb + mb) * kHeads * 128 + h * 128 + c;
    const float *ml = p.part_ml + static_cast<int64_t>(row) * p.nsplit * 2 * kHeads;
    float4 v[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int su = sub + ws * u;
      v[u] = (su < p.nsplit) ? *reinterpret_cast<const float4 *>(po + su * sstride)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const int s0 = lane, s1 = lane + 32;
    const float m0 = (s0 < p.nsplit) ? ml[s0 * 2 * kHeads + h] : -INFINITY;
    const float m1 = (s1 < p.nsplit) ? ml[s1 * 2 * kHeads + h] : -INFINITY;
    const float l0 = (s0 < p.nsplit) ? ml[s0 * 2 * kHeads + kHeads + h] : 0.f;
    const float l1 = (s1 < p.nsplit) ? ml[s1 * 2 * kHeads + kHeads + h] : 0.f;
    float M = fmaxf(m0, m1);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float e0 = (m0 == -INFINITY) ? 0.f : exp2f(m0 - M);
    const float e1 = (m1 == -INFINITY) ? 0.f : exp2f(m1 - M);
    float L = e0 * l0 + e1 * l1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    const float il = (L > 0.f) ? 1.f / L : 0.f;
    const float w0 = e0 * il, w1 = e1 * il;  // normalised merge weights of splits lane, lane+32
    if (sub == 0 && lane == 0 && mb == 0)
      p.lse[static_cast<int64_t>(row) * p.H + h] = (L > 0.f) ? (M + log2f(L)) * kLn2 : -INFINITY;
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int su = sub + ws * u;  // warp-uniform
      if (su < p.nsplit) {
        const float w = __shfl_sync(0xffffffffu, su < 32 ? w0 : w1, su & 31);
        acc.x += w * v[u].x; acc.y += w * v[u].y; acc.z += w * v[u].z; acc.w += w * v[u].w;
      }
    }
  }
  if (ws > 1) {
    part[warp][lane] = acc;
    __syncthreads();
    if (sub == 0) {
      for (int q = 1; q < ws; ++q) {
        const float4 b = part[warp + q][lane];
        acc.x += b.x; acc.y += b.y; acc.z += b.z; acc.w += b.w;
      }
    }
  }
  const int r = mb * 128 + c;
  if (active && sub == 0 && r < p.R) {
    float *dst = p.out + (static_cast<int64_t>(row) * p.H + h) * p.R + r;  // 4-byte aligned only
    dst[0] = acc.x;
    dst[1] = acc.y;
    dst[2] = acc.z;
    dst[3] = acc.w;
  }
}

// ---------------------------------------------------------------------------
// Pipelined variant: the latent tile is a ring of two 64-key halves, filled
// and consumed by different warps at once.
//
//   warps 0-7   softmax of each half (the four warps whose TMEM lane quadrant
//               holds the half's keys, each for 32 heads), the rare rescale of
//               the O accumulator (all eight, one quadrant and head half each),
//               and the epilogue
//   warps 8-11  gather: two groups of two warps, group g filling half-slot g
//               (halves g, g + 2, ...) with 16-byte cp.async pieces of the
//               selected rows; each group waits for its own copies and posts
//               the slot, so two halves can be in flight at once
//   warp 12     one thread issues tcgen05.mma: S(j) as soon as half j has
//               landed, PV(j) as soon as its probabilities are written, in
//               whichever order they become ready
//
// S(j) = L . Q^T runs over all 128 rows of the tile (M = 128; the other
// half's rows are ignored) into one of two TMEM S buffers, so the logits of
// half j + 1 are computed while half j's softmax runs.  P(j) = hi + lo (two
// bf16 terms, near-fp32 weights): the hi term is written over half j's rows
// of the first atom the PV product never reads (the rope atom at R = 512),
// which S(j) has finished with; the lo term goes to one 8 KB buffer, free once
// PV(j - 1) has completed.  A tcgen05.mma instruction costs about the same
// time for N = 64 heads as for N = 256 (measured), so the kernel is bound by
// its instruction count.
// ---------------------------------------------------------------------------
constexpr int kPipeThreads = 416;
constexpr int kPipeSoftWarps = 8;
constexpr int kPipeProdWarp0 = 8;
constexpr int kPipeMmaWarp = 12;
constexpr int kHalfKeys = 64;
constexpr int kPipeMisc = 1664;

struct PipeLayout {
  int nQ, nmb, ap;  // query atoms, 128-column PV blocks, atom holding P hi
  uint32_t off_q, off_lo, off_misc, bytes;
};
__host__ __device__ inline PipeLayout pipe_layout(int R, int P) {
  PipeLayout l;
  const int W = R + P;
  l.nQ = (W + 63) / 64;
  l.nmb = (R + 127) / 128;
  const int nL = l.nQ > 2 * l.nmb ? l.nQ : 2 * l.nmb;
  l.ap = (nL > 2 * l.nmb) ? 2 * l.nmb : nL;  // first atom PV never reads
  const int nLa = nL > l.ap ? nL : l.ap + 1;
  l.off_q = static_cast<uint32_t>(nLa) * kAtomL;
  l.off_lo = l.off_q + static_cast<uint32_t>(l.nQ) * kAtomQ;
  l.off_misc = l.off_lo + 64 * 128;
  l.bytes = l.off_misc + kPipeMisc;
  return l;
}

// barrier over `n` threads that also returns whether any of them passed true
__device__ __forceinline__ bool named_bar_or(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(n)
      : "memory");
  return r != 0u;
}
// bounded wait that also gives up as soon as another role has failed
__device__ __forceinline__ bool pipe_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns,
                                          volatile uint32_t *failed) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*failed) return false;
    if (global_timer_ns() - t0 > limit_ns) {
      *failed = 1u;
      return false;
    }
  }
}

// kLat8: the latent cache holds E4M3 rows with one fp32 scale per token.  The
// gather stages each row's 64-byte E4M3 slice of an atom in the upper half of
// its 128-byte destination row (cp.async), then widens it in place to bf16;
// the token's scale multiplies its logit and its PV weight (the dequantized
// row is scale * e4m3(code)).
template <bool kClusterMerge, bool kLat8>
__global__ void __launch_bounds__(kPipeThreads, 1) mla_pipe_kernel(const MlaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const PipeLayout lay = pipe_layout(p.R, p.W - p.R);
  const int W = p.W, R = p.R, nQ = lay.nQ, nmb = lay.nmb;
  uint8_t *Ls = smem;
  uint8_t *Qs = smem + lay.off_q;
  uint8_t *Lo = smem + lay.off_lo;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + lay.off_misc);
  uint64_t *full = bars;        // [2] half-slot landed (one arrive per producer warp)
  uint64_t *empty = bars + 2;   // [2] PV of the slot's half completed (MMA commit)
  uint64_t *sfull = bars + 4;   // [2] S of the slot's half in TMEM (MMA commit)
  uint64_t *pready = bars + 6;  // P of the current half written (one arrive per softmax warp)
  uint64_t *qready = bars + 7;  // query tile landed (one arrive per softmax warp)
  uint64_t *bar_drain = bars + 8;
  uint64_t *bar_stall = bars + 9;
  // [0] TMEM base, [1] failed
  uint32_t *misc = reinterpret_cast<uint32_t *>(bars + 10);
  volatile uint32_t *failed = misc + 1;
  uint32_t *vmask = misc + 4;                           // [slot][producer warp] valid keys
  float *red = reinterpret_cast<float *>(vmask + 4);    // [2][64]
  float *mrun = red + 2 * kHeads;                       // [64] running max (log2 units)
  float *alpha = mrun + kHeads;                         // [64] rescale of this half
  float *kscale = alpha + kHeads;                       // [2][64] per-key scale (kLat8)

  const int tid = threadIdx.x, warp = warp_id(), lane = lane_id();
  const int split = blockIdx.x;
  // causal rows grow with t: start the longest ones first
  const int row = p.causal ? (p.n_q - 1 - static_cast<int>(blockIdx.y)) : static_cast<int>(blockIdx.y);
  const int b = p.causal ? 0 : row;
  const int cpr = W / 8;  // 16-byte pieces per row

  // TMEM: the logits of half-slot s at columns 64 s, O^T from column 128
  uint32_t tmem_cols = 32;
  while (tmem_cols < static_cast<uint32_t>(2 * kHeads + nmb * kHeads)) tmem_cols <<= 1;
  if (tid == 0) {
    mbar_init(&full[0], 2);
    mbar_init(&full[1], 2);
    mbar_init(&empty[0], 1);
    mbar_init(&empty[1], 1);
    mbar_init(&sfull[0], 1);
    mbar_init(&sfull[1], 1);
    mbar_init(pready, kPipeSoftWarps);
    mbar_init(qready, kPipeSoftWarps);
    mbar_init(bar_drain, 1);
    mbar_init(bar_stall, 1);
    misc[1] = 0u;
    fence_barrier_init();
  }
  if (tid < kHeads) mrun[tid] = -INFINITY;
  if (warp == kPipeMmaWarp) {
    tmem_alloc(&misc[0], tmem_cols);
    tmem_relinquish();
  }
  // softmax warps: the 64-head query tile (heads >= H zero-filled),
  // 128B-swizzled, K-major; before the dependency wait when q predates the
  // kernel in front of this one
  auto load_q = [&]() {
    const uint16_t *qrow = p.q + static_cast<int64_t>(row) * p.H * W;
    const uint32_t qs = smem_u32(Qs);
    for (int h = warp; h < kHeads; h += kPipeSoftWarps) {
      const bool ok = h < p.H;
      for (int cc = lane; cc < cpr; cc += 32) {
        const uint16_t *src = ok ? qrow + h * W + cc * 8 : p.q;
        cp_async_16(qs + (cc >> 3) * kAtomQ + h * 128 + (((cc & 7) ^ (h & 7)) << 4), src,
                    ok ? 16u : 0u);
      }
    }
    cp_async_commit();
  };
  if (p.early_q && warp < kPipeSoftWarps) load_q();
  griddep_wait();
  if (!p.early_q && warp < kPipeSoftWarps) load_q();
  griddep_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  if (p.debug_stall) {
    if (tid == 0 && !mbar_wait(bar_stall, 0u, p.wait_ns)) *failed = 1u;
    __syncthreads();
  }

  // this CTA's halves: the row keeps at most min(topk, len) tokens, in its
  // first slots
  const int len = p.causal ? p.q_pos0 + row + 1 : p.seq_lens[b];
  const int limit = min(len, p.max_pages * kPageSize);
  const int nsel = max(0, min(p.topk, len));
  const int nh_row = (nsel + kHalfKeys - 1) / kHalfKeys;
  const int h_begin = split * p.chunks_per_split;
  const int nh = max(0, min(nh_row, h_begin + p.chunks_per_split) - h_begin);

  float lpart = 0.f;  // softmax warps: sum of p for head 32 hh + lane over this quadrant's keys

  if (warp < kPipeSoftWarps) {
    // ------------------------------------------------------------ softmax
    const int q4 = warp & 3, hh = warp >> 2;
    cp_async_wait_all();
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(qready);
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const int prow = 32 * q4 + lane;                  // this thread's tile row (key slot)
    const uint32_t p_hi = smem_u32(Ls + lay.ap * kAtomL) + prow * 128;
    const int lrow = 32 * (q4 & 1) + lane;            // its row of the lo buffer
    const uint32_t p_lo = smem_u32(Lo) + lrow * 128;
    // every exit from this loop is decided by a reduction over all eight
    // warps (named_bar_or), so they always take the same number of barriers
    for (int j = 0; j < nh; ++j) {
      const int s = j & 1;
      const uint32_t par = (j >> 1) & 1;
      const bool active = (q4 >> 1) == s;
      bool ok = pipe_wait(&sfull[s], par, p.wait_ns, failed) &&
                pipe_wait(&full[s], par, p.wait_ns, failed);
      tc_fence_after();
      float z[32];
      if (ok && active) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + lane_off + 64 * s + 32 * hh, v);
        tmem_ld_wait();
        const bool kvalid = (vmask[s * 2 + (q4 & 1)] >> lane) & 1u;
        // (FP8 rows: the logit of the dequantized row, the key's scale applied)
        const float zs = kLat8 ? p.scale_log2 * kscale[s * kHalfKeys + 32 * (q4 & 1) + lane]
                               : p.scale_log2;
#pragma unroll
        for (int i = 0; i < 32; ++i) z[i] = kvalid ? __uint_as_float(v[i]) * zs : -INFINITY;
        red[(q4 & 1) * kHeads + 32 * hh + lane] = butterfly32<true>([&](int i) { return z[i]; });
      }
      if (named_bar_or(1, 32 * kPipeSoftWarps, !ok)) break;
      bool need = false;
      if (tid < kHeads) {
        const float mc = fmaxf(red[tid], red[kHeads + tid]);
        const float m_old = mrun[tid];
        const float m_new = (mc > m_old + kRescaleLog2) ? mc : m_old;
        const float a = (m_new == m_old) ? 1.f : exp2f(m_old - m_new);
        alpha[tid] = a;
        mrun[tid] = m_new;
        need = (a != 1.f) && j > 0;
      }
      const bool rescale = named_bar_or(1, 32 * kPipeSoftWarps, need);
      // PV(j - 1) must be complete: the lo buffer is reused and, on a
      // rescale, the O accumulator must hold every earlier half
      bool ok2 = true;
      if (j > 0) ok2 = pipe_wait(&empty[(j - 1) & 1], ((j - 1) >> 1) & 1, p.wait_ns, failed);
      if (ok2) {
        tc_fence_after();
        if (rescale) {
          for (int mi = 0; mi < nmb; ++mi) {
            const uint32_t ta = tmem + lane_off + 2 * kHeads + mi * kHeads + 32 * hh;
            uint32_t v[32];
            tmem_ld_32x32b_x32(ta, v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i)
              v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha[32 * hh + i]);
            tmem_st_32x32b_x32(ta, v);
          }
          tmem_st_wait();
        }
        float psum = 0.f;
        if (active) {
          // p in fp32 (its sum is l); the PV weight is p rounded to fp16
#pragma unroll
          for (int i = 0; i < 32; ++i)
            z[i] = (z[i] == -INFINITY) ? 0.f : exp2f(z[i] - mrun[32 * hh + i]);
          psum = butterfly32<false>([&](int i) { return z[i]; });
          // the PV weight (p, or for FP8 rows p times the key's scale) as
          // hi + lo, two bf16 terms: near-fp32 weights
          const float wk = kLat8 ? kscale[s * kHalfKeys + 32 * (q4 & 1) + lane] : 1.f;
          uint32_t phi[16], plo[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float p0 = z[2 * i] * wk, p1 = z[2 * i + 1] * wk;
            const __nv_bfloat162 hi = __floats2bfloat162_rn(p0, p1);
            const __nv_bfloat162 lo =
                __floats2bfloat162_rn(p0 - __low2float(hi), p1 - __high2float(hi));
            phi[i] = *reinterpret_cast<const uint32_t *>(&hi);
            plo[i] = *reinterpret_cast<const uint32_t *>(&lo);
          }
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const uint32_t u = static_cast<uint32_t>(((4 * hh + jj) ^ (prow & 7)) << 4);
            st_shared_v4(p_hi + u, make_uint4(phi[4 * jj], phi[4 * jj + 1], phi[4 * jj + 2], phi[4 * jj + 3]));
            st_shared_v4(p_lo + u, make_uint4(plo[4 * jj], plo[4 * jj + 1], plo[4 * jj + 2], plo[4 * jj + 3]));
          }
        }
        lpart = lpart * alpha[32 * hh + lane] + psum;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      if (named_bar_or(1, 32 * kPipeSoftWarps, !ok2)) break;
      if (lane == 0) mbar_arrive(pready);
    }
    // the last PV must be complete before O is read
    if (!*failed && nh > 0)
      pipe_wait(&empty[(nh - 1) & 1], ((nh - 1) >> 1) & 1, p.wait_ns, failed);
  } else if (warp < kPipeMmaWarp) {
    // ------------------------------------------------------------ gather
    const int g = (warp - kPipeProdWarp0) >> 1;  // half-slot this group fills
    const int wl = (warp - kPipeProdWarp0) & 1;  // rows 32 wl .. of the half
    const int jj = lane & 7;                     // 16-byte piece within each 128-byte atom row
    const uint32_t ls = smem_u32(Ls);
    // resolve the selected position of slot (h_begin + j) * 64 + 32 wl + lane
    auto resolve = [&](int j) -> int {
      if (j >= nh) return -1;
      const int slot = (h_begin + j) * kHalfKeys + 32 * wl + lane;
      if (slot >= nsel) return -1;
      const int pos = p.idx[static_cast<int64_t>(row) * p.topk + slot];
      if (pos < 0) return -1;
      if (pos >= limit) {
        report(p.status, kErrBadIndex, (kKernMla << 24) | (slot & 0xFFFF));
        return -1;
      }
      const int page = p.block_table[static_cast<int64_t>(b) * p.max_pages + pos / kPageSize];
      if (page < 0 || page >= p.num_pages) {
        report(p.status, kErrBadPage, (kKernMla << 24) | (slot & 0xFFFF));
        return -1;
      }
      return page * kPageSize + pos % kPageSize;
    };
    int phys = resolve(g);
    for (int j = g; j < nh; j += 2) {
      const int u = j >> 1;
      if (u >= 1 && !pipe_wait(&empty[g], (u - 1) & 1, p.wait_ns, failed)) break;
      const uint32_t mask = __ballot_sync(0xffffffffu, phys >= 0);
      if (lane == 0) vmask[g * 2 + wl] = mask;
      if constexpr (kLat8) {
        // E4M3: quarter jq (16 bytes) of each atom's 64-byte slice, staged in
        // physical 16-byte unit 4 + jq of the row's 128-byte destination
        const int jq = lane & 3, rr = lane >> 2;
#pragma unroll 1
        for (int k = 0; k < 4; ++k) {
          const int rk = rr + 8 * k;
          const int ph = __shfl_sync(0xffffffffu, phys, rk);
          const int trow = kHalfKeys * g + 32 * wl + rk;
          const uint32_t stg = ls + trow * 128 + 64 + 16 * jq;
          const uint8_t *src = p.latent8 + static_cast<int64_t>(ph < 0 ? 0 : ph) * W + 16 * jq;
          for (int a = 0; a < nQ; ++a) {
            const bool ok = ph >= 0 && a * 64 + 16 * jq < W;
            cp_async_16(stg + a * kAtomL, ok ? src + a * 64 : p.latent8, ok ? 16u : 0u);
          }
        }
      } else {
#pragma unroll 2
        for (int k = 0; k < 8; ++k) {
          const int rk = (lane >> 3) + 4 * k;            // row within this warp's 32
          const int ph = __shfl_sync(0xffffffffu, phys, rk);
          const int trow = kHalfKeys * g + 32 * wl + rk;  // tile row
          const uint32_t dst = ls + trow * 128 + ((jj ^ (trow & 7)) << 4);
          const uint16_t *src = p.latent + static_cast<int64_t>(ph < 0 ? 0 : ph) * W + jj * 8;
          for (int a = 0; a < nQ; ++a) {
            const bool ok = ph >= 0 && a * 8 + jj < cpr;
            cp_async_16(dst + a * kAtomL, ok ? src + a * 64 : p.latent, ok ? 16u : 0u);
          }
        }
      }
      cp_async_commit();
      // the scale of each of this warp's rows (a key-less slot: 0, so that its
      // weight is 0 rather than 0 times whatever the slot holds)
      if constexpr (kLat8)
        kscale[g * kHalfKeys + 32 * wl + lane] = (phys >= 0) ? p.lat_scale[phys] : 0.f;
      const int phys_next = resolve(j + 2);  // overlaps the copies in flight
      cp_async_wait_all();
      if constexpr (kLat8) {
        // widen in place (the four quarters of a row are lanes of this warp)
        const int jq = lane & 3, rr = lane >> 2;
#pragma unroll 1
        for (int k = 0; k < 4; ++k) {
          const int trow = kHalfKeys * g + 32 * wl + rr + 8 * k;
          widen_e4m3_quarter(ls + trow * 128, static_cast<uint32_t>(trow & 7), jq, nQ);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[g]);
      phys = phys_next;
    }
    cp_async_wait_all();
  } else if (lane == 0) {
    // ------------------------------------------------------------ MMA issue
    const uint32_t idesc_s = idesc_bf16_f32(kChunk, kHeads, 0, 0);
    const uint32_t idesc_pv = idesc_bf16_f32(kChunk, kHeads, 1, 1);
    const uint32_t ls = smem_u32(Ls), qs = smem_u32(Qs), lo = smem_u32(Lo);
    const uint32_t phb = ls + lay.ap * kAtomL;
    // descriptors at the tiles' bases; an operand at byte offset o adds o >> 4
    // to the start-address field (no carry: shared addresses stay below 2^18)
    const uint64_t d_l = smem_desc(ls, 16, 1024, kLayoutSW128);        // L, K-major
    const uint64_t d_q = smem_desc(qs, 16, 1024, kLayoutSW128);        // Q, K-major
    const uint64_t d_v = smem_desc(ls, kAtomL, 1024, kLayoutSW128);    // L as V^T, MN-major
    const uint64_t d_hi = smem_desc(phb, kAtomQ, 1024, kLayoutSW128);  // P hi, MN-major
    const uint64_t d_lo = smem_desc(lo, kAtomQ, 1024, kLayoutSW128);   // P lo, MN-major
    bool ok = nh == 0 || pipe_wait(qready, 0u, p.wait_ns, failed);
    // S(ns) as soon as its half has landed (at most one ahead of the PV
    // products), PV(npv) as soon as its weights are written
    int ns = 0, npv = 0;
    uint64_t t0 = global_timer_ns();
    uint32_t spins = 0;
    while (ok && npv < nh) {
      bool progressed = false;
      if (ns < nh && ns <= npv + 1 && mbar_try_wait(&full[ns & 1], (ns >> 1) & 1)) {
        fence_proxy_async_smem();
        tc_fence_after();
        const uint32_t d = tmem + 64 * (ns & 1);
        for (int a = 0; a < nQ; ++a)
          for (int kk = 0; kk < 4; ++kk) {
            if (a * 64 + kk * 16 >= W) break;
            mma_bf16(d, d_l + ((a * kAtomL + kk * 32) >> 4), d_q + ((a * kAtomQ + kk * 32) >> 4),
                     idesc_s, (a | kk) != 0 ? 1u : 0u);
          }
        mma_commit(&sfull[ns & 1]);
        ++ns;
        progressed = true;
      }
      if (npv < ns && mbar_try_wait(pready, npv & 1)) {
        tc_fence_after();
        const int s = npv & 1;
        for (int mi = 0; mi < nmb; ++mi)
          for (int part = 0; part < 2; ++part)
            for (int ks = 0; ks < 4; ++ks) {
              const uint32_t krow = static_cast<uint32_t>(kHalfKeys * s + 16 * ks) * 128;
              const uint64_t b = part ? d_lo + ((16 * ks * 128) >> 4) : d_hi + (krow >> 4);
              mma_bf16(tmem + 2 * kHeads + mi * kHeads, d_v + ((2 * mi * kAtomL + krow) >> 4), b,
                       idesc_pv, (npv > 0 || part || ks) ? 1u : 0u);
            }
        mma_commit(&empty[s]);
        ++npv;
        progressed = true;
      }
      if (progressed) {
        t0 = global_timer_ns();
        spins = 0;
      } else if (++spins >= 64) {
        spins = 0;
        if (*failed) ok = false;
        else if (global_timer_ns() - t0 > p.wait_ns) {
          *failed = 1u;
          ok = false;
        }
      }
    }
    if (*failed) {
      mma_commit(bar_drain);  // fires once every MMA issued above has completed
      mbar_wait(bar_drain, 0u, kDrainLimitNs);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const bool bad = *failed != 0u;
  if (bad && tid == 0) report(p.status, kErrTimeout, (kKernMla << 24) | 1u);
  const bool have_o = !bad && nh > 0;
  // the row sum of p over the four lane quadrants (the query tile is free)
  float *lred = reinterpret_cast<float *>(Qs);  // [4][64]
  const int q4 = warp & 3, hh = (warp >> 2) & 1;
  if (warp < kPipeSoftWarps) lred[q4 * kHeads + 32 * hh + lane] = have_o ? lpart : 0.f;
  __syncthreads();
  float *lsum = red;           // [64]
  float *rinv = red + kHeads;  // [64]
  if (tid < kHeads) {
    lsum[tid] = (lred[tid] + lred[kHeads + tid]) + (lred[2 * kHeads + tid] + lred[3 * kHeads + tid]);
    if (!have_o) {
      mrun[tid] = -INFINITY;
      lsum[tid] = 0.f;
    }
  }
  __syncthreads();
  const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
  const uint32_t tmem_o = tmem + 2 * kHeads;

  if constexpr (kClusterMerge) {
    // The row's splits are the CTAs of this cluster.  Once every CTA is past
    // its loop (first barrier), each sends its (m, l) to every CTA, then its
    // O^T, scaled to the common maximum, in 32-column units (32 latent
    // columns x 64 heads, 8 KB) to the unit's owner (unit u = 4 mb + quadrant,
    // owner u % C), into the owner's latent tile.  An owner sums its units
    // over the C senders and writes the output.
    const uint32_t C = cluster_nctarank(), me = cluster_ctarank();
    float *ml_all = reinterpret_cast<float *>(Lo);  // [C][2][64]
    cluster_sync();
    if (tid < 2 * kHeads) {
      const int h = tid & (kHeads - 1);
      const float v = (tid < kHeads) ? mrun[h] : lsum[h];
      const uint32_t a = smem_u32(&ml_all[(me * 2 + (tid >> 6)) * kHeads + h]);
      for (uint32_t r = 0; r < C; ++r) st_dsmem_u32(map_to_rank(a, r), __float_as_uint(v));
    }
    cluster_sync();
    if (tid < kHeads) {
      float M = -INFINITY;
      for (uint32_t r = 0; r < C; ++r) M = fmaxf(M, ml_all[(r * 2) * kHeads + tid]);
      float L = 0.f;
      for (uint32_t r = 0; r < C; ++r) {
        const float m = ml_all[(r * 2) * kHeads + tid];
        if (m != -INFINITY) L += exp2f(m - M) * ml_all[(r * 2 + 1) * kHeads + tid];
      }
      alpha[tid] = (mrun[tid] == -INFINITY) ? 0.f : exp2f(mrun[tid] - M);
      rinv[tid] = (L > 0.f) ? 1.f / L : 0.f;
      if (me == 0 && tid < p.H)
        p.lse[static_cast<int64_t>(row) * p.H + tid] = (L > 0.f) ? (M + log2f(L)) * kLn2 : -INFINITY;
    }
    __syncthreads();
    const uint32_t recv = smem_u32(Ls);  // [units / C][C senders][32 columns][64 heads]
    if (warp < kPipeSoftWarps) {
      for (int mb = 0; mb < nmb; ++mb) {
        uint32_t v[32];
        if (have_o) {
          tmem_ld_32x32b_x32(tmem_o + lane_off + mb * kHeads + 32 * hh, v);
          tmem_ld_wait();
        }
#pragma unroll
        for (int i = 0; i < 32; ++i)
          v[i] = have_o ? __float_as_uint(__uint_as_float(v[i]) * alpha[32 * hh + i]) : 0u;
        const uint32_t u = static_cast<uint32_t>(mb * 4 + q4);
        const uint32_t owner = u % C, slot = (u / C) * C + me;
        const uint32_t base = recv + (slot * 2048u + lane * 64u) * 4u;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t hsw = static_cast<uint32_t>((32 * hh + 4 * k) ^ ((lane & 7) << 2));
          st_dsmem_v4(map_to_rank(base + hsw * 4u, owner), v[4 * k], v[4 * k + 1], v[4 * k + 2],
                      v[4 * k + 3]);
        }
      }
    }
    cluster_sync();  // every unit is in its owner's buffer; no remote access follows
    if (warp < kPipeSoftWarps) {
      const float *rbuf = reinterpret_cast<const float *>(Ls);
      const uint32_t nunits = static_cast<uint32_t>(nmb * 4);
      for (uint32_t j = 0; j * C + me < nunits; ++j) {
        const uint32_t u = j * C + me;
        const int col = static_cast<int>(u >> 2) * 128 + static_cast<int>(u & 3) * 32 + lane;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int g = warp + 8 * k;  // heads 4g .. 4g+3
          const int hsw = (4 * g) ^ ((lane & 7) << 2);
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
          for (uint32_t src = 0; src < C; ++src) {
            const float4 x =
                *reinterpret_cast<const float4 *>(rbuf + ((j * C + src) * 2048u + lane * 64 + hsw));
            acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
          }
          const float a4[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int h = 4 * g + i;
            if (h < p.H && col < R)
              p.out[(static_cast<int64_t>(row) * p.H + h) * R + col] = a4[i] * rinv[h];
          }
        }
      }
    }
  } else if (p.nsplit == 1) {
    // the whole selection ran here: normalise and write the output
    if (warp < kPipeSoftWarps) {
      for (int mi = 0; mi < nmb; ++mi) {
        uint32_t v[32];
        if (have_o) {
          tmem_ld_32x32b_x32(tmem_o + lane_off + mi * kHeads + 32 * hh, v);
          tmem_ld_wait();
        }
        const int r = mi * 128 + q4 * 32 + lane;
        if (r < R) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int h = 32 * hh + i;
            if (h >= p.H) break;
            const float l = lsum[h];
            const float o = (have_o && l > 0.f) ? __uint_as_float(v[i]) / l : 0.f;
            p.out[(static_cast<int64_t>(row) * p.H + h) * R + r] = o;
          }
        }
      }
    }
    if (tid < p.H) {
      const float l = lsum[tid];
      p.lse[static_cast<int64_t>(row) * p.H + tid] =
          (l > 0.f) ? (mrun[tid] + log2f(l)) * kLn2 : -INFINITY;
    }
  } else {
    // partial (m, l, O) of this split for the merge kernel; O^T leaves one
    // 128-column block at a time through shared memory (the latent tile is
    // free) with a bulk asynchronous store
    float *Obuf = reinterpret_cast<float *>(Ls);
    float *dst = p.part_o + (static_cast<int64_t>(row) * p.nsplit + split) * nmb * kHeads * 128;
    if (tid < kHeads) {
      float *ml = p.part_ml + (static_cast<int64_t>(row) * p.nsplit + split) * 2 * kHeads;
      ml[tid] = mrun[tid];
      ml[kHeads + tid] = lsum[tid];
    }
    for (int mi = 0; mi < nmb; ++mi) {
      float *blk = Obuf + mi * kHeads * 128;
      if (warp < kPipeSoftWarps) {
        uint32_t v[32];
        if (have_o) {
          tmem_ld_32x32b_x32(tmem_o + lane_off + mi * kHeads + 32 * hh, v);
          tmem_ld_wait();
        }
        const int cc = q4 * 32 + lane;
#pragma unroll
        for (int i = 0; i < 32; ++i) blk[(32 * hh + i) * 128 + cc] = have_o ? __uint_as_float(v[i]) : 0.f;
        fence_proxy_async_smem();
      }
      __syncthreads();
      if (tid == 0) {
        asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                         reinterpret_cast<uint64_t>(dst + mi * kHeads * 128)),
                     "r"(smem_u32(blk)), "r"(static_cast<uint32_t>(kHeads * 128 * 4))
                     : "memory");
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      }
    }
    if (tid == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kPipeMmaWarp) {
    __syncwarp();
    tmem_dealloc(tmem, tmem_cols);
  }
}

size_t mla_smem_bytes(int R, int P) {
  const int W = R + P;
  const int nQ = (W + 63) / 64;
  const int nmb = (R + 127) / 128;
  const int nL = std::max(nQ, 2 * nmb);
  const bool p_overlays = nL > 2 * nmb;
  return 1024 + static_cast<size_t>(nL) * kAtomL + (p_overlays ? 0 : kAtomL) +
         static_cast<size_t>(nQ) * kAtomQ + 4 * kChunk + 4 * (7 * kHeads) +
         8 * 4 + 16 + 4 * (kMaxMergeCluster * 2 * kHeads) + 4 * kChunk;
}

struct SplitPlan {
  int nsplit, chunks_per_split, merge, kc;
};

SplitPlan plan_splits(int n_q, int topk) {
  // with few rows, 64-key chunks put twice as many SMs on the gathers
  const int kc = (static_cast<int64_t>(n_q) * ((topk + kChunk - 1) / kChunk) <
                  device_sm_count() / 2) ? 64 : kChunk;
  const int nchunks = (topk + kc - 1) / kc;
  int want = (device_sm_count() + n_q - 1) / std::max(1, n_q);
  want = std::max(1, std::min(want, std::min(nchunks, 64)));
  const int cps = (nchunks + want - 1) / want;
  const int ns = (nchunks + cps - 1) / cps;
  SplitPlan s;
  s.nsplit = ns;
  s.chunks_per_split = cps;
  s.merge = (ns == 1) ? kMergeNone : kMergeGlobal;
  s.kc = kc;
  return s;
}

size_t pipe_smem_bytes(int R, int P) { return 1024 + pipe_layout(R, P).bytes; }

// whether clusters of `size` pipelined CTAs can be co-scheduled on this device
// (queried once per size and device)
bool pipe_cluster_ok(int size, size_t smem) {
  static int cached[64][17];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64 || size < 2 || size > 16)
    return false;
  if (cached[dev][size] == 0) {
    // both latent formats share the launch shape; the query uses the bf16 one
    bool ok = true;
    for (const void *k : {reinterpret_cast<const void *>(mla_pipe_kernel<true, false>),
                          reinterpret_cast<const void *>(mla_pipe_kernel<true, true>)}) {
      ok = ok && func_attr_once(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(device_max_smem_optin())) == cudaSuccess;
      if (ok && size > 8)
        ok = func_attr_once(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
    }
    if (ok) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(size, 1, 1);
      cfg.blockDim = dim3(kPipeThreads, 1, 1);
      cfg.dynamicSmemBytes = smem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = size;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      const cudaError_t qe = cudaOccupancyMaxActiveClusters(&n, mla_pipe_kernel<true, false>, &cfg);
      if (qe != cudaSuccess) note_cuda_error(qe, "cluster occupancy query");
      ok = qe == cudaSuccess && n > 0;
    }
    cudaGetLastError();  // clear a rejected query
    cached[dev][size] = ok ? 1 : -1;
  }
  return cached[dev][size] > 0;
}

// How the pipelined kernel lays a batch over CTAs.  A row's halves (64 keys
// each) are split over CTAs only while the rows leave SMs idle, keeping at
// least two halves per CTA so that the gather of one overlaps the other's
// arithmetic.  Up to 16 splits that divide the row's 32-column units merge in
// one cluster through distributed shared memory; more go through global
// scratch and the merge kernel.
struct PipePlan {
  int nsplit, hps, cluster;  // splits per row, halves per split, cluster merge
};
PipePlan plan_pipe(int n_q, int topk, int R, int P) {
  const int nh = (topk + kHalfKeys - 1) / kHalfKeys;
  const int sms = device_sm_count();
  const int units = 4 * ((R + 127) / 128);
  PipePlan pl{1, nh, 0};
  if (n_q >= sms) return pl;
  const int target = std::min(std::max(1, sms / std::max(1, n_q)), std::max(1, nh / 2));
  if (target <= 1) return pl;
  if (target <= 16) {
    const size_t smem = pipe_smem_bytes(R, P);
    for (int c = target; c >= 2; --c)
      if (units % c == 0 && pipe_cluster_ok(c, smem)) {
        pl.nsplit = c;
        pl.hps = (nh + c - 1) / c;
        pl.cluster = 1;
        return pl;
      }
  }
  const int ns = std::min(target, 64);
  pl.hps = (nh + ns - 1) / ns;
  pl.nsplit = (nh + pl.hps - 1) / pl.hps;
  return pl;
}

// The pipelined kernel when the batch's 64-key halves fill at least two waves
// of SMs (many rows, or prefill); with fewer, the per-chunk kernel, which
// spreads a few rows over more SMs (one CTA per 128-column block of the output).
bool use_pipe(int n_q, int topk) {
  const int64_t halves = static_cast<int64_t>(n_q) * ((topk + kHalfKeys - 1) / kHalfKeys);
  return halves >= 2 * static_cast<int64_t>(device_sm_count());
}

}  // namespace

int mla_num_splits(int n_q, int topk) { return plan_splits(n_q, topk).nsplit; }

size_t mla_pipe_scratch_bytes(int n_q, int topk, int R) {
  // the widest latent row a call may use (R + P <= 576) only changes the
  // cluster query's shared-memory size, which the pipelined kernel always fits
  const PipePlan pl = plan_pipe(n_q, topk, R, 576 - R);
  if (pl.nsplit == 1 || pl.cluster) return 0;
  const size_t o = static_cast<size_t>(n_q) * pl.nsplit * ((R + 127) / 128) * kHeads * 128 * 4;
  const size_t ml = static_cast<size_t>(n_q) * pl.nsplit * 2 * kHeads * 4;
  return ((o + 255) & ~static_cast<size_t>(255)) + ml;
}
namespace {
size_t chunk_scratch_bytes(int n_q, int topk, int R) {
  const SplitPlan s = plan_splits(n_q, topk);
  if (s.merge != kMergeGlobal) return 0;
  const size_t o = static_cast<size_t>(n_q) * s.nsplit * ((R + 127) / 128) * kHeads * 128 * 4;
  const size_t ml = static_cast<size_t>(n_q) * s.nsplit * 2 * kHeads * 4;
  return ((o + 255) & ~static_cast<size_t>(255)) + ml;
}
}  // namespace

// enough for either latent format (both take the same kernel for a shape)
size_t mla_scratch_bytes(int n_q, int topk, int R) {
  const size_t pipe = mla_pipe_scratch_bytes(n_q, topk, R);
  return use_pipe(n_q, topk) ? pipe : std::max(pipe, chunk_scratch_bytes(n_q, topk, R));
}

// whether clusters of `size` MLA CTAs with `smem` bytes each can be co-scheduled
// (queried once per size and device)
bool mla_cluster_ok(int size, size_t smem) {
  static int cached[64][kMaxMergeCluster + 1];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64 || size < 2 ||
      size > kMaxMergeCluster)
    return false;
  if (cached[dev][size] == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(size, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = size;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    const bool ok =
        cudaOccupancyMaxActiveClusters(&n, mla_kernel<true, false>, &cfg) == cudaSuccess && n > 0;
    cudaGetLastError();  // clear a rejected query
    cached[dev][size] = ok ? 1 : -1;
  }
  return cached[dev][size] > 0;
}

int mla_launch_count(int n_q, int topk, int R, int P, bool /*lat8: the same kernels*/) {
  if (use_pipe(n_q, topk)) {
    const PipePlan pl = plan_pipe(n_q, topk, R, P);
    return (pl.nsplit == 1 || pl.cluster) ? 1 : 2;
  }
  const SplitPlan sp = plan_splits(n_q, topk);
  if (sp.merge != kMergeGlobal) return 1;
  const int nmb = (R + 127) / 128;
  const int ncb = (nmb > 1 && static_cast<int64_t>(n_q) * sp.nsplit * nmb <= device_sm_count()) ? nmb : 1;
  const bool cluster = ncb == 1 && sp.nsplit <= kMaxMergeCluster && (nmb * 4) % sp.nsplit == 0 &&
                       mla_cluster_ok(sp.nsplit, mla_smem_bytes(R, P));
  return cluster ? 1 : 2;
}

template <bool L8>
dsa_status_t launch_mla_pipe(const MlaLaunch &a, cudaStream_t stream) {
  const size_t smem = pipe_smem_bytes(a.R, a.P);
  if (smem > device_max_smem_optin()) return DSA_ERR_UNSUPPORTED;
  for (const void *k : {reinterpret_cast<const void *>(mla_pipe_kernel<false, L8>),
                        reinterpret_cast<const void *>(mla_pipe_kernel<true, L8>)})
    if (func_attr_once(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       static_cast<int>(device_max_smem_optin())) != cudaSuccess)
      return DSA_ERR_CUDA;
  const PipePlan pl = plan_pipe(a.n_q, a.topk, a.R, a.P);
  const int nmb = (a.R + 127) / 128;
  MlaParams p;
  p.q = a.q;
  p.latent = a.latent;
  p.latent8 = a.latent8;
  p.lat_scale = a.lat_scale;
  p.idx = a.idx;
  p.seq_lens = a.seq_lens;
  p.block_table = a.block_table;
  p.out = a.out;
  p.lse = a.lse;
  p.part_o = nullptr;
  p.part_ml = nullptr;
  const bool global = pl.nsplit > 1 && !pl.cluster;
  if (global) {
    const size_t o = static_cast<size_t>(a.n_q) * pl.nsplit * nmb * kHeads * 128 * 4;
    const size_t need = ((o + 255) & ~static_cast<size_t>(255)) +
                        static_cast<size_t>(a.n_q) * pl.nsplit * 2 * kHeads * 4;
    if (a.scratch == nullptr || a.scratch_bytes < need) return DSA_ERR_WORKSPACE;
    p.part_o = static_cast<float *>(a.scratch);
    p.part_ml = reinterpret_cast<float *>(static_cast<uint8_t *>(a.scratch) +
                                          ((o + 255) & ~static_cast<size_t>(255)));
  }
  p.n_q = a.n_q;
  p.H = a.H;
  p.R = a.R;
  p.W = a.R + a.P;
  p.topk = a.topk;
  p.causal = a.causal;
  p.q_pos0 = a.q_pos0;
  p.max_pages = a.max_pages;
  p.num_pages = a.num_pages;
  p.nsplit = pl.nsplit;
  p.chunks_per_split = pl.hps;
  p.kc = kHalfKeys;
  p.ncb = 1;
  p.comb_ws = 1;
  p.cluster_merge = pl.cluster;
  p.scale_log2 = static_cast<float>(static_cast<double>(a.scale) * 1.4426950408889634);
  p.wait_ns = wait_limit_ns();
  p.debug_stall = debug_stall() == kKernMla ? 1 : 0;
  p.early_q = a.early_q;
  p.status = a.status;
  const cudaError_t le =
      pl.cluster ? launch_pdl(mla_pipe_kernel<true, L8>, dim3(pl.nsplit, a.n_q, 1), dim3(kPipeThreads),
                              smem, stream, static_cast<unsigned>(pl.nsplit), p)
                 : launch_pdl(mla_pipe_kernel<false, L8>, dim3(pl.nsplit, a.n_q, 1),
                              dim3(kPipeThreads), smem, stream, 1u, p);
  if (le != cudaSuccess) return DSA_ERR_CUDA;
  if (global) {
    p.comb_ws = pl.nsplit > 16 ? 4 : (pl.nsplit > 8 ? 2 : 1);
    const int blocks_per_cta = kCombineWarps / p.comb_ws;
    if (launch_pdl(combine_kernel, dim3(a.n_q, a.H, (nmb + blocks_per_cta - 1) / blocks_per_cta),
                   dim3(32 * kCombineWarps), 0, stream, 1, p) != cudaSuccess)
      return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

// the per-chunk kernel for a few rows (bf16 or E4M3 latent rows)
template <bool L8>
dsa_status_t launch_mla_chunk(const MlaLaunch &a, cudaStream_t stream) {
  const int W = a.R + a.P;
  const size_t smem = mla_smem_bytes(a.R, a.P);
  if (smem > device_max_smem_optin()) return DSA_ERR_UNSUPPORTED;
  for (const void *k : {reinterpret_cast<const void *>(mla_kernel<false, L8>),
                        reinterpret_cast<const void *>(mla_kernel<true, L8>)})
    if (func_attr_once(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       static_cast<int>(device_max_smem_optin())) != cudaSuccess)
      return DSA_ERR_CUDA;
  const SplitPlan sp = plan_splits(a.n_q, a.topk);
  MlaParams p;
  p.q = a.q;
  p.latent = a.latent;
  p.latent8 = a.latent8;
  p.lat_scale = a.lat_scale;
  p.idx = a.idx;
  p.seq_lens = a.seq_lens;
  p.block_table = a.block_table;
  p.out = a.out;
  p.lse = a.lse;
  p.part_o = nullptr;
  p.part_ml = nullptr;
  if (sp.merge == kMergeGlobal) {
    const size_t o =
        static_cast<size_t>(a.n_q) * sp.nsplit * ((a.R + 127) / 128) * kHeads * 128 * 4;
    const size_t need = ((o + 255) & ~static_cast<size_t>(255)) +
                        static_cast<size_t>(a.n_q) * sp.nsplit * 2 * kHeads * 4;
    if (a.scratch == nullptr || a.scratch_bytes < need) return DSA_ERR_WORKSPACE;
    p.part_o = static_cast<float *>(a.scratch);
    p.part_ml = reinterpret_cast<float *>(static_cast<uint8_t *>(a.scratch) +
                                          ((o + 255) & ~static_cast<size_t>(255)));
  }
  p.n_q = a.n_q;
  p.H = a.H;
  p.R = a.R;
  p.W = W;
  p.topk = a.topk;
  p.causal = a.causal;
  p.q_pos0 = a.q_pos0;
  p.max_pages = a.max_pages;
  p.num_pages = a.num_pages;
  p.nsplit = sp.nsplit;
  p.chunks_per_split = sp.chunks_per_split;
  p.kc = sp.kc;
  p.scale_log2 = static_cast<float>(static_cast<double>(a.scale) * 1.4426950408889634);
  p.wait_ns = wait_limit_ns();
  p.debug_stall = debug_stall() == kKernMla ? 1 : 0;
  p.early_q = a.early_q;
  p.status = a.status;
  // few CTAs: one per 128-column block of the output as well, when that still fits one wave
  const int nmb = (a.R + 127) / 128;
  p.ncb = (nmb > 1 && static_cast<int64_t>(a.n_q) * sp.nsplit * nmb <= device_sm_count()) ? nmb : 1;
  p.comb_ws = 1;
  // a row split over 2..8 CTAs that divide its 32-column units merges inside
  // one cluster, when the device co-schedules such clusters
  p.cluster_merge = (sp.merge == kMergeGlobal && p.ncb == 1 && sp.nsplit <= kMaxMergeCluster &&
                     (nmb * 4) % sp.nsplit == 0 && mla_cluster_ok(sp.nsplit, smem))
                        ? 1 : 0;
  const cudaError_t le =
      p.cluster_merge
          ? launch_pdl(mla_kernel<true, L8>, dim3(sp.nsplit, a.n_q, p.ncb), dim3(kThreads), smem,
                       stream, static_cast<unsigned>(sp.nsplit), p)
          : launch_pdl(mla_kernel<false, L8>, dim3(sp.nsplit, a.n_q, p.ncb), dim3(kThreads), smem,
                       stream, 1u, p);
  if (le != cudaSuccess) return DSA_ERR_CUDA;
  if (sp.merge == kMergeGlobal && !p.cluster_merge) {
    // warps per column block: enough that each loads at most eight splits
    p.comb_ws = sp.nsplit > 16 ? 4 : (sp.nsplit > 8 ? 2 : 1);
    const int blocks_per_cta = kCombineWarps / p.comb_ws;
    if (launch_pdl(combine_kernel,
                   dim3(a.n_q, a.H, (nmb + blocks_per_cta - 1) / blocks_per_cta),
                   dim3(32 * kCombineWarps), 0, stream, 1, p) != cudaSuccess)
      return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

dsa_status_t launch_mla(const MlaLaunch &a, cudaStream_t stream) {
  const bool l8 = a.latent8 != nullptr;
  if (a.force_pipe || use_pipe(a.n_q, a.topk))
    return l8 ? launch_mla_pipe<true>(a, stream) : launch_mla_pipe<false>(a, stream);
  return l8 ? launch_mla_chunk<true>(a, stream) : launch_mla_chunk<false>(a, stream);
}

}  // namespace dsa
