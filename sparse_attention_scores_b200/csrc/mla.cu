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
// Design (sm_100a): a CTA of 4 warps owns one query row and a contiguous range
// of 128-key chunks of its selection.  The 64-head absorbed query stays in
// shared memory for the whole range.  Per chunk:
//   gather   the 128 selected latent rows (1,152 B each at R+P = 576) with
//            16-byte cp.async into a 128B-swizzled K-major tile; unused slots
//            are zero-filled
//   S^T      tcgen05.mma, M = 128 keys, N = 64 heads, K = R + P, into TMEM
//   softmax  one thread per key holds its 64 logits; per-head max and sum
//            over the 128 keys by a transposing butterfly of warp shuffles;
//            the running max moves only when it grows by more than 2^8, and
//            then the TMEM accumulator is rescaled
//   O^T     += tcgen05.mma, M = 128 latent columns (R/128 blocks), N = 64
//            heads, K = 128 keys; the same shared tile serves as V^T
//            (MN-major view), P is written as bf16 over the rope atom
// PV uses p = hi + lo (two bf16 terms) for near-fp32 weights.
// A row split over several CTAs writes (m, l, O) partials that a second
// kernel merges by log-sum-exp weights.
#include <algorithm>
#include <cuda_bf16.h>
#include <math.h>

#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kThreads = 128;
constexpr int kChunk = 128;   // keys per chunk = MMA M
constexpr int kHeads = 64;    // head columns of every tile = MMA N
constexpr int kAtomL = kChunk * 128;  // bytes of one 64-column atom of the latent tile
constexpr int kAtomQ = kHeads * 128;  // bytes of one 64-column atom of the query tile
constexpr float kRescaleLog2 = 8.0f;

struct MlaParams {
  const uint16_t *q;
  const uint16_t *latent;
  const int32_t *idx;
  const int32_t *seq_lens;
  const int32_t *block_table;
  float *out;
  float *lse;
  float *part_o;   // [n_q, nsplit, 64, R]
  float *part_ml;  // [n_q, nsplit, 2, 64]
  int n_q, H, R, W, topk, causal, q_pos0, max_pages, num_pages;
  int nsplit, chunks_per_split;
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

// Reduce 64 per-key values over the 32 keys (lanes) of a warp, for every head
// at once.  Each butterfly step halves the heads a lane keeps and exchanges
// the other half with its partner; afterwards lane L holds the reductions of
// heads 2L and 2L+1 in o[0], o[1].  62 shuffles instead of 64 x 5.
template <bool kMax, typename Get>
__device__ __forceinline__ void butterfly64(Get v, float (&o)[2]) {
  const int lane = lane_id();
  auto op = [](float a, float b) { return kMax ? fmaxf(a, b) : a + b; };
  float a[32];
  {
    const bool up = lane & 16;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float lo_h = v(i), hi_h = v(i + 32);
      const float send = up ? lo_h : hi_h;
      const float keep = up ? hi_h : lo_h;
      a[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 16));
    }
  }
  float b[16];
  {
    const bool up = lane & 8;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float send = up ? a[i] : a[i + 16];
      const float keep = up ? a[i + 16] : a[i];
      b[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 8));
    }
  }
  float c[8];
  {
    const bool up = lane & 4;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float send = up ? b[i] : b[i + 8];
      const float keep = up ? b[i + 8] : b[i];
      c[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 4));
    }
  }
  float d[4];
  {
    const bool up = lane & 2;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float send = up ? c[i] : c[i + 4];
      const float keep = up ? c[i + 4] : c[i];
      d[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 2));
    }
  }
  {
    const bool up = lane & 1;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float send = up ? d[i] : d[i + 2];
      const float keep = up ? d[i + 2] : d[i];
      o[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 1));
    }
  }
}

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
  const uint16_t **rowp = reinterpret_cast<const uint16_t **>(Qs + nQ * kAtomQ);  // [128]
  float *red = reinterpret_cast<float *>(rowp + kChunk);  // [4][64]
  float *mrun = red + 4 * kHeads;
  float *lrun = mrun + kHeads;
  float *alpha = lrun + kHeads;
  uint64_t *bars = reinterpret_cast<uint64_t *>(alpha + kHeads);  // [0] S done, [1] PV done, [2] drain
  uint32_t *misc = reinterpret_cast<uint32_t *>(bars + 4);        // [0] tmem, [1] rescale, [2] failed

  const int tid = threadIdx.x, warp = warp_id(), lane = lane_id();
  const int split = blockIdx.x, row = blockIdx.y;
  const int b = p.causal ? 0 : row;
  const int nchunks = (p.topk + kChunk - 1) / kChunk;
  const int c_begin = split * p.chunks_per_split;
  const int c_end = min(nchunks, c_begin + p.chunks_per_split);
  const int cpr = W / 8;  // 16-byte pieces per latent row

  uint32_t tmem_cols = 32;
  while (tmem_cols < static_cast<uint32_t>(kHeads + nmb * kHeads)) tmem_cols <<= 1;
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    mbar_init(&bars[2], 1);
    mbar_init(&bars[3], 1);
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
    // warp w copies heads w, w+4, ...; its lanes walk the 16-byte pieces of a row
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
  if (p.early_q) griddep_wait();
  griddep_launch_dependents();
  const int limit = min(p.causal ? p.q_pos0 + row + 1 : p.seq_lens[b], p.max_pages * kPageSize);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_s = misc[0];
  const uint32_t tmem_o = misc[0] + kHeads;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t idesc_s = idesc_bf16_f32(kChunk, kHeads, 0, 0);
  const uint32_t idesc_pv = idesc_bf16_f32(kChunk, kHeads, 1, 1);
  uint32_t phase = 0, pv_phase = 0;
  bool have_o = false;
  bool failed = false;

  if (p.debug_stall) {
    if (!mbar_wait(&bars[3], 0u, p.wait_ns)) misc[2] = 1u;
    __syncthreads();
    if (misc[2]) failed = true;
  }
  for (int ch = c_begin; ch < c_end && !failed; ++ch) {
    // resolve the 128 selected positions of this chunk
    {
      const int slot = ch * kChunk + tid;
      int pos = (slot < p.topk) ? p.idx[static_cast<int64_t>(row) * p.topk + slot] : -1;
      const uint16_t *src = nullptr;
      if (pos >= 0) {
        if (pos >= limit) {
          report(p.status, kErrBadIndex, (kKernMla << 24) | (slot & 0xFFFF));
        } else {
          const int page = p.block_table[static_cast<int64_t>(b) * p.max_pages + pos / kPageSize];
          if (page < 0 || page >= p.num_pages)
            report(p.status, kErrBadPage, (kKernMla << 24) | (slot & 0xFFFF));
          else
            src = p.latent + (static_cast<int64_t>(page) * kPageSize + pos % kPageSize) * W;
        }
      }
      rowp[tid] = src;
      if (tid == 0) misc[1] = 0u;
    }
    __syncthreads();
    // gather the latent rows (invalid slots are zero-filled)
    {
      const uint32_t ls = smem_u32(Ls);
      for (int key = warp; key < kChunk; key += kThreads / 32) {
        const uint16_t *src = rowp[key];
        for (int cc = lane; cc < cpr; cc += 32)
          cp_async_16(ls + (cc >> 3) * kAtomL + key * 128 + (((cc & 7) ^ (key & 7)) << 4),
                      src ? src + cc * 8 : p.latent, src ? 16u : 0u);
      }
      cp_async_commit();
      cp_async_wait_all();
      fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // S^T = L . Q^T  (M = 128 keys, N = 64 heads, K = W)
    if (tid == 0) {
      const uint32_t ls = smem_u32(Ls), qs = smem_u32(Qs);
      for (int a = 0; a < nQ; ++a)
        for (int kk = 0; kk < 4; ++kk) {
          if (a * 64 + kk * 16 >= W) break;
          mma_bf16(tmem_s, smem_desc(ls + a * kAtomL + kk * 32, 16, 1024, kLayoutSW128),
                   smem_desc(qs + a * kAtomQ + kk * 32, 16, 1024, kLayoutSW128), idesc_s,
                   (a | kk) != 0 ? 1u : 0u);
        }
      mma_commit(&bars[0]);
    }
    if (!mbar_wait(&bars[0], phase, p.wait_ns)) {
      failed = true;
      misc[2] = 1u;
    }
    tc_fence_after();
    __syncthreads();
    if (misc[2]) { failed = true; break; }

    // logits of key (warp*32 + lane), log2 units
    const bool kvalid = rowp[tid] != nullptr;
    float z[64];
    {
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem_s + lane_off, v);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) z[i] = kvalid ? __uint_as_float(v[i]) * p.scale_log2 : -INFINITY;
      tmem_ld_32x32b_x32(tmem_s + lane_off + 32, v);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i)
        z[32 + i] = kvalid ? __uint_as_float(v[i]) * p.scale_log2 : -INFINITY;
    }
    // per-head chunk max over the 128 keys
    {
      float o[2];
      butterfly64<true>([&](int h) { return z[h]; }, o);
      red[warp * kHeads + 2 * lane] = o[0];
      red[warp * kHeads + 2 * lane + 1] = o[1];
    }
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
    uint32_t phi[32], plo[32];  // packed bf16 pairs of heads (2i, 2i+1)
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int h = 2 * i;
      const float p0 = (z[h] == -INFINITY) ? 0.f : exp2f(z[h] - mrun[h]);
      const float p1 = (z[h + 1] == -INFINITY) ? 0.f : exp2f(z[h + 1] - mrun[h + 1]);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(p0, p1);
      const __nv_bfloat162 lo =
          __floats2bfloat162_rn(p0 - __low2float(hi), p1 - __high2float(hi));
      phi[i] = *reinterpret_cast<const uint32_t *>(&hi);
      plo[i] = *reinterpret_cast<const uint32_t *>(&lo);
    }
    {
      // p of head h as the PV product sees it: hi + lo
      auto pf = [&](int h) {
        const uint32_t a = phi[h >> 1], b = plo[h >> 1];
        const uint32_t ha = (h & 1) ? (a & 0xFFFF0000u) : (a << 16);
        const uint32_t hb = (h & 1) ? (b & 0xFFFF0000u) : (b << 16);
        return __uint_as_float(ha) + __uint_as_float(hb);
      };
      float o[2];
      butterfly64<false>(pf, o);
      red[warp * kHeads + 2 * lane] = o[0];
      red[warp * kHeads + 2 * lane + 1] = o[1];
    }
    __syncthreads();
    if (tid < kHeads) {
      const float lc = (red[tid] + red[kHeads + tid]) + (red[2 * kHeads + tid] + red[3 * kHeads + tid]);
      lrun[tid] = lrun[tid] * alpha[tid] + lc;
    }
    // rescale the O accumulator when some head's running max moved
    if (misc[1]) {
      for (int mb = 0; mb < nmb; ++mb)
        for (int half = 0; half < 2; ++half) {
          const uint32_t ta = tmem_o + lane_off + mb * kHeads + half * 32;
          uint32_t v[32];
          tmem_ld_32x32b_x32(ta, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i)
            v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha[half * 32 + i]);
          tmem_st_32x32b_x32(ta, v);
        }
      tmem_st_wait();
    }
    // O^T += L^T . P^T  (M = 128 latent columns per block, N = 64 heads), in two
    // halves of 64 keys; each half multiplies by the hi and by the lo terms.
    // The 16 KB P region holds [hi | lo] for the 64 keys of one half.
    bool pv_failed = false;
    for (int half = 0; half < 2; ++half) {
      if ((warp >> 1) == half) {
        const int rk = tid & 63;
        const uint32_t base = smem_u32(Ps) + rk * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t off = ((j ^ (rk & 7)) << 4);
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
        for (int mb = 0; mb < nmb; ++mb)
          for (int part = 0; part < 2; ++part)
            for (int ks = 0; ks < 4; ++ks)
              mma_bf16(tmem_o + mb * kHeads,
                       smem_desc(ls + 2 * mb * kAtomL + (half * 4 + ks) * 2048, kAtomL, 1024,
                                 kLayoutSW128),
                       smem_desc(ps + part * 8192 + ks * 2048, kAtomQ, 1024, kLayoutSW128),
                       idesc_pv, (have_o || half || part || ks) ? 1u : 0u);
        mma_commit(&bars[1]);
      }
      if (!mbar_wait(&bars[1], pv_phase, p.wait_ns)) misc[2] = 1u;
      pv_phase ^= 1u;
      tc_fence_after();
      __syncthreads();
      if (misc[2]) { pv_failed = true; break; }
    }
    if (pv_failed) failed = true;
    have_o = true;
    phase ^= 1u;
  }
  cp_async_wait_all();

  if (failed) {
    if (tid == 0) {
      report(p.status, kErrTimeout, (kKernMla << 24) | 1u);
      mma_commit(&bars[2]);  // fires once every MMA issued above has completed
      mbar_wait(&bars[2], 0u, kDrainLimitNs);
    }
  } else {
    // write the normalised output (single split) or the partial (m, l, O)
    const bool direct = p.nsplit == 1;
    for (int mb = 0; mb < nmb; ++mb)
      for (int half = 0; half < 2; ++half) {
        uint32_t v[32];
        if (have_o) {
          tmem_ld_32x32b_x32(tmem_o + lane_off + mb * kHeads + half * 32, v);
          tmem_ld_wait();
        }
        const int r = mb * 128 + warp * 32 + lane;
        if (r < R) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int h = half * 32 + i;
            if (h >= p.H) break;
            const float o = have_o ? __uint_as_float(v[i]) : 0.f;
            if (direct) {
              const float l = lrun[h];
              p.out[(static_cast<int64_t>(row) * p.H + h) * R + r] = (l > 0.f) ? o / l : 0.f;
            } else {
              p.part_o[((static_cast<int64_t>(row) * p.nsplit + split) * kHeads + h) * R + r] = o;
            }
          }
        }
      }
    if (tid < p.H) {
      if (direct) {
        const float l = lrun[tid];
        p.lse[static_cast<int64_t>(row) * p.H + tid] =
            (l > 0.f) ? (mrun[tid] + log2f(l)) * 0.69314718055994531f : -INFINITY;
      } else {
        float *ml = p.part_ml + (static_cast<int64_t>(row) * p.nsplit + split) * 2 * kHeads;
        ml[tid] = mrun[tid];
        ml[kHeads + tid] = lrun[tid];
      }
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

// Merge the split partials of one (row, head):
//   out = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s,  lse = (M + log2 L) ln 2.
// The first warp loads every split's (m, l) in parallel (nsplit <= 64) and
// reduces them with shuffles; all threads then stream the partial rows.
__global__ void __launch_bounds__(128) combine_kernel(const MlaParams p) {
  const int row = blockIdx.x, h = blockIdx.y;
  griddep_wait();
  griddep_launch_dependents();
  const float *ml = p.part_ml + static_cast<int64_t>(row) * p.nsplit * 2 * kHeads;
  __shared__ float wgt[64];
  __shared__ float inv_l;
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int s0 = lane, s1 = lane + 32;
    const float m0 = (s0 < p.nsplit) ? ml[s0 * 2 * kHeads + h] : -INFINITY;
    const float m1 = (s1 < p.nsplit) ? ml[s1 * 2 * kHeads + h] : -INFINITY;
    const float l0 = (s0 < p.nsplit) ? ml[s0 * 2 * kHeads + kHeads + h] : 0.f;
    const float l1 = (s1 < p.nsplit) ? ml[s1 * 2 * kHeads + kHeads + h] : 0.f;
    float M = fmaxf(m0, m1);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float w0 = (m0 == -INFINITY) ? 0.f : exp2f(m0 - M);
    const float w1 = (m1 == -INFINITY) ? 0.f : exp2f(m1 - M);
    float L = w0 * l0 + w1 * l1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    wgt[s0] = w0;
    wgt[s1] = w1;
    if (lane == 0) {
      inv_l = (L > 0.f) ? 1.f / L : 0.f;
      p.lse[static_cast<int64_t>(row) * p.H + h] =
          (L > 0.f) ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
    }
  }
  __syncthreads();
  const float il = inv_l;
  const float *po = p.part_o + (static_cast<int64_t>(row) * p.nsplit * kHeads + h) * p.R;
  const int64_t sstride = static_cast<int64_t>(kHeads) * p.R;
  for (int r = threadIdx.x; r < p.R; r += blockDim.x) {
    float acc = 0.f;
#pragma unroll 8
    for (int s = 0; s < p.nsplit; ++s) acc += wgt[s] * po[s * sstride + r];
    p.out[(static_cast<int64_t>(row) * p.H + h) * p.R + r] = acc * il;
  }
}

}  // namespace

int mla_num_splits(int n_q, int topk) {
  const int nchunks = (topk + kChunk - 1) / kChunk;
  int want = (device_sm_count() + n_q - 1) / std::max(1, n_q);
  want = std::max(1, std::min(want, std::min(nchunks, 64)));
  const int cps = (nchunks + want - 1) / want;
  return (nchunks + cps - 1) / cps;
}

size_t mla_scratch_bytes(int n_q, int topk, int R) {
  const int ns = mla_num_splits(n_q, topk);
  if (ns <= 1) return 0;
  const size_t o = static_cast<size_t>(n_q) * ns * kHeads * R * 4;
  const size_t ml = static_cast<size_t>(n_q) * ns * 2 * kHeads * 4;
  return ((o + 255) & ~static_cast<size_t>(255)) + ml;
}

dsa_status_t launch_mla(const MlaLaunch &a, cudaStream_t stream) {
  const int W = a.R + a.P;
  const int nQ = (W + 63) / 64;
  const int nmb = (a.R + 127) / 128;
  const int nL = std::max(nQ, 2 * nmb);
  const bool p_overlays = nL > 2 * nmb;
  const size_t smem = 1024 + static_cast<size_t>(nL) * kAtomL + (p_overlays ? 0 : kAtomL) +
                      static_cast<size_t>(nQ) * kAtomQ + 8 * kChunk + 4 * (7 * kHeads) + 32 + 16;
  if (smem > device_max_smem_optin()) return DSA_ERR_UNSUPPORTED;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(device_max_smem_optin())) != cudaSuccess)
      return DSA_ERR_CUDA;
    attr_set = true;
  }
  const int nchunks = (a.topk + kChunk - 1) / kChunk;
  const int nsplit = mla_num_splits(a.n_q, a.topk);
  const int cps = (nchunks + nsplit - 1) / nsplit;
  MlaParams p;
  p.q = a.q;
  p.latent = a.latent;
  p.idx = a.idx;
  p.seq_lens = a.seq_lens;
  p.block_table = a.block_table;
  p.out = a.out;
  p.lse = a.lse;
  p.part_o = nullptr;
  p.part_ml = nullptr;
  if (nsplit > 1) {
    if (a.scratch == nullptr || a.scratch_bytes < mla_scratch_bytes(a.n_q, a.topk, a.R))
      return DSA_ERR_WORKSPACE;
    const size_t o = static_cast<size_t>(a.n_q) * nsplit * kHeads * a.R * 4;
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
  p.nsplit = nsplit;
  p.chunks_per_split = cps;
  p.scale_log2 = static_cast<float>(static_cast<double>(a.scale) * 1.4426950408889634);
  p.wait_ns = wait_limit_ns();
  p.debug_stall = debug_stall() == kKernMla ? 1 : 0;
  p.early_q = a.early_q;
  p.status = a.status;
  if (launch_pdl(mla_kernel, dim3(nsplit, a.n_q), dim3(kThreads), smem, stream, 1, p) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  if (nsplit > 1) {
    if (launch_pdl(combine_kernel, dim3(a.n_q, a.H), dim3(128), 0, stream, 1, p) != cudaSuccess)
      return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

}  // namespace dsa
