// The absorption GEMMs around the step: the absorbed query in front of it and
// the value projection after the split merge.
//
//   q_abs[b, h, 0:R]     = q_nope[b, h, :] . W_UK[h]        (bf16 out)
//   q_abs[b, h, R:R+P]   = q_rope[b, h, :]
//   v_out[b, h, :]       = o_lat[b, h, :] . W_UV[h]          (fp32 out)
//
// ("Self-contained GLM-5 serving stack: Just Vx kernels compiled to PTX",
// file list: absorbed MLA decode over compressed request-local KV, i.e. the
// up-projections are folded into the query and applied to the output instead
// of to every cached row; "GLM on an A100, in Vx", "The model": one latent
// vector per token serves as key and value.)
//
// Design (sm_100a): one CTA per (head, 128-row tile of the output features,
// tile of batch rows).  Both products are D^T = W^T . X^T, so the weight tile
// is the A operand (M = 128 output features, MN-major: the weight's rows are
// the K index and its 128 columns lie contiguous in memory, loaded by TMA
// with 128-byte swizzle) and the activations are the B operand (N = batch
// rows, K-major, staged by the CTA's threads).  The fp32 value input of the
// projection enters as two bf16 terms (hi + lo, like the attention weights of
// the PV product), so the projection keeps near-fp32 inputs.  One thread issues
// the tcgen05.mma chain into tensor memory; four warps read the 128 lanes
// back and write rows of the output.
#include <cuda_bf16.h>

#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kThreads = 128;
constexpr int kTileM = 128;            // output features per CTA
constexpr int kAtomCols = 64;          // weight columns per 128-byte swizzle atom
constexpr int kMaxBoxRows = 256;       // TMA box height limit

struct AbsorbParams {
  const uint16_t *x;      // absorb: q_nope [n, H, K]; (project uses xf)
  const float *xf;        // project: o_lat [n, H, K] fp32
  const uint16_t *rope;   // absorb: q_rope [n, H, P] (nullptr when P == 0)
  uint16_t *out_bf16;     // absorb: q_abs [n, H, M + P]
  float *out_f32;         // project: v_out [n, H, M]
  int n, H, K, M, P;      // rows, heads, reduction length, output features, rope width
  int n_tile;             // batch rows per CTA (multiple of 16, <= 256)
  uint64_t wait_ns;
  DevStatus *status;
};

__device__ __forceinline__ void tmem_ld_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// kProject = false: the absorbed query; true: the value projection.
template <bool kProject>
__global__ void __launch_bounds__(kThreads, 1)
    absorb_kernel(const __grid_constant__ CUtensorMap tmW, const AbsorbParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const int K = p.K, NT = p.n_tile;
  const int a_atom = K * 128;                 // bytes of one 64-column weight atom
  const int b_atom = NT * 128;                // bytes of one 64-wide K atom of the activations
  const int nkb = K / 64;                     // K atoms of the activations
  uint8_t *As = smem;                         // [2 atoms][K rows][128 B]
  uint8_t *Bs = As + 2 * a_atom;              // [terms][nkb atoms][NT rows][128 B]
  uint64_t *bar_a = reinterpret_cast<uint64_t *>(Bs + (kProject ? 2 : 1) * nkb * b_atom);
  uint64_t *bar_mma = bar_a + 1;
  uint32_t *misc = reinterpret_cast<uint32_t *>(bar_mma + 1);  // [0] tmem base, [1] failed

  const int tid = threadIdx.x, warp = warp_id(), lane = lane_id();
  const int n0 = blockIdx.x * NT, mt = blockIdx.y, h = blockIdx.z;
  const int m0 = mt * kTileM;
  uint32_t tmem_cols = 32;
  while (tmem_cols < static_cast<uint32_t>(NT)) tmem_cols <<= 1;

  if (tid == 0) {
    mbar_init(bar_a, 1);
    mbar_init(bar_mma, 1);
    misc[1] = 0u;
    fence_barrier_init();
    tma_prefetch_desc(&tmW);
  }
  if (warp == 0) { tmem_alloc(&misc[0], tmem_cols); tmem_relinquish(); }
  __syncthreads();
  // the activations (and, in general, the weights) may come from earlier work
  griddep_wait();
  griddep_launch_dependents();

  // A: weight rows [h*K, h*K + K) (the K index), columns [m0, m0 + 128) in two
  // 64-column atoms, boxes of at most 256 rows
  if (tid == 0) {
    mbar_arrive_expect_tx(bar_a, static_cast<uint32_t>(2 * a_atom));
    for (int j = 0; j < 2; ++j)
      for (int r0 = 0; r0 < K; r0 += kMaxBoxRows)
        tma_load_2d(As + j * a_atom + r0 * 128, &tmW, m0 + j * kAtomCols, h * K + r0, bar_a);
  }
  // B: batch rows n0 .. n0 + NT of head h, K-major, 128-byte swizzled; rows
  // past n are zero
  if (!kProject) {
    const uint32_t bs = smem_u32(Bs);
    const int pieces = NT * (K / 8);  // 16-byte pieces
    for (int pc = tid; pc < pieces; pc += kThreads) {
      const int r = pc / (K / 8), c = pc - r * (K / 8);
      const int b = n0 + r;
      const bool ok = b < p.n;
      const uint16_t *src = ok ? p.x + (static_cast<int64_t>(b) * p.H + h) * K + c * 8 : p.x;
      cp_async_16(bs + (c >> 3) * b_atom + r * 128 + (((c & 7) ^ (r & 7)) << 4), src, ok ? 16u : 0u);
    }
    cp_async_commit();
    cp_async_wait_all();
  } else {
    // fp32 inputs as hi + lo bf16 terms: 16 bytes (eight values) of each term
    // per piece
    const int pieces = NT * (K / 8);
    for (int pc = tid; pc < pieces; pc += kThreads) {
      const int r = pc / (K / 8), c = pc - r * (K / 8);
      const int b = n0 + r;
      float v[8];
      if (b < p.n) {
        const float4 *src =
            reinterpret_cast<const float4 *>(p.xf + (static_cast<int64_t>(b) * p.H + h) * K + c * 8);
        const float4 x0 = src[0], x1 = src[1];
        v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w;
        v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.f;
      }
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 a = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        const __nv_bfloat162 e =
            __floats2bfloat162_rn(v[2 * i] - __low2float(a), v[2 * i + 1] - __high2float(a));
        hi[i] = *reinterpret_cast<const uint32_t *>(&a);
        lo[i] = *reinterpret_cast<const uint32_t *>(&e);
      }
      const uint32_t off = (c >> 3) * b_atom + r * 128 + (((c & 7) ^ (r & 7)) << 4);
      const uint32_t dh = smem_u32(Bs) + off, dl = smem_u32(Bs) + nkb * b_atom + off;
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dh), "r"(hi[0]), "r"(hi[1]),
                   "r"(hi[2]), "r"(hi[3])
                   : "memory");
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dl), "r"(lo[0]), "r"(lo[1]),
                   "r"(lo[2]), "r"(lo[3])
                   : "memory");
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  if (tid == 0) {
    bool ok = mbar_wait(bar_a, 0u, p.wait_ns);
    if (ok) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16_f32(kTileM, NT, 1, 0);
      const uint32_t as = smem_u32(As), bs = smem_u32(Bs);
      const int terms = kProject ? 2 : 1;
      for (int t = 0; t < terms; ++t)
        for (int ks = 0; ks < K / 16; ++ks)
          mma_bf16(tmem,
                   smem_desc(as + ks * 2048, a_atom, 1024, kLayoutSW128),  // 16 K rows per step
                   smem_desc(bs + t * nkb * b_atom + (ks >> 2) * b_atom + (ks & 3) * 32, 16, 1024,
                             kLayoutSW128),
                   idesc, (t | ks) != 0 ? 1u : 0u);
    } else {
      misc[1] = 1u;
      report(p.status, kErrTimeout, (kKernAbsorb << 24) | (kProject ? 2u : 1u));
      mbar_wait(bar_a, 0u, kDrainLimitNs);  // let the loads land before the memory goes away
    }
    mma_commit(bar_mma);
  }
  if (!mbar_wait(bar_mma, 0u, p.wait_ns)) misc[1] = 1u;
  tc_fence_after();
  __syncthreads();
  if (misc[1] == 0u) {
    // lane 32*warp + i of the accumulator is output feature m0 + 32*warp + i;
    // column j is batch row n0 + j
    const int f = m0 + 32 * warp + lane;
    const uint32_t lane_off = static_cast<uint32_t>(32 * warp) << 16;
    for (int c0 = 0; c0 < NT && n0 + c0 < p.n; c0 += 16) {
      uint32_t v[16];
      tmem_ld_x16(tmem + lane_off + c0, v);
      tmem_ld_wait();
      if (f < p.M) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int b = n0 + c0 + i;
          if (b >= p.n) break;
          const int64_t row = static_cast<int64_t>(b) * p.H + h;
          if (kProject)
            p.out_f32[row * p.M + f] = __uint_as_float(v[i]);
          else
            p.out_bf16[row * (p.M + p.P) + f] =
                __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[i])));
        }
      }
    }
  }
  // the rope part passes through unchanged (one feature tile does it)
  if (!kProject && mt == 0 && p.P > 0) {
    const int pieces = NT * (p.P / 8);
    for (int pc = tid; pc < pieces; pc += kThreads) {
      const int r = pc / (p.P / 8), c = pc - r * (p.P / 8);
      const int b = n0 + r;
      if (b >= p.n) continue;
      const int64_t row = static_cast<int64_t>(b) * p.H + h;
      *reinterpret_cast<uint4 *>(p.out_bf16 + row * (p.M + p.P) + p.M + c * 8) =
          *reinterpret_cast<const uint4 *>(p.rope + row * p.P + c * 8);
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

size_t absorb_smem(int K, int n_tile, bool project) {
  return 1024 + 2 * static_cast<size_t>(K) * 128 +
         (project ? 2 : 1) * static_cast<size_t>(K / 64) * n_tile * 128 + 16 + 16;
}

template <bool kProject>
dsa_status_t launch_absorb_impl(const AbsorbLaunch &a, cudaStream_t stream) {
  const int K = a.K;
  // batch rows per CTA: as many as shared memory allows, at most 256
  int nt = 256;
  while (nt > 16 && absorb_smem(K, nt, kProject) > device_max_smem_optin()) nt /= 2;
  if (absorb_smem(K, nt, kProject) > device_max_smem_optin()) return DSA_ERR_UNSUPPORTED;
  if (a.n <= 128) nt = std::min(nt, std::max(16, (a.n + 15) / 16 * 16));
  if (func_attr_once(reinterpret_cast<const void *>(absorb_kernel<kProject>),
                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                     static_cast<int>(device_max_smem_optin())) != cudaSuccess)
    return DSA_ERR_CUDA;
  CUtensorMap tmW;
  // the weights as [H * K rows][M columns]; boxes of 64 columns x min(K, 256) rows
  if (!make_map_2d(&tmW, a.w, static_cast<uint64_t>(a.M), static_cast<uint64_t>(a.H) * K, 64,
                   std::min(K, kMaxBoxRows), 128))
    return DSA_ERR_CUDA;
  AbsorbParams p;
  p.x = a.x;
  p.xf = a.xf;
  p.rope = a.rope;
  p.out_bf16 = a.out_bf16;
  p.out_f32 = a.out_f32;
  p.n = a.n;
  p.H = a.H;
  p.K = K;
  p.M = a.M;
  p.P = a.P;
  p.n_tile = nt;
  p.wait_ns = wait_limit_ns();
  p.status = a.status;
  // a last feature tile of 64 reads its upper 64 weight columns out of bounds
  // (zero fill, 128-byte aligned start) and does not write them
  const dim3 grid(static_cast<unsigned>((a.n + nt - 1) / nt),
                  static_cast<unsigned>((a.M + kTileM - 1) / kTileM),
                  static_cast<unsigned>(a.H));
  if (launch_pdl(absorb_kernel<kProject>, grid, dim3(kThreads), absorb_smem(K, nt, kProject),
                 stream, 1, tmW, p) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

}  // namespace

dsa_status_t launch_absorb(const AbsorbLaunch &a, cudaStream_t stream) {
  return a.project ? launch_absorb_impl<true>(a, stream) : launch_absorb_impl<false>(a, stream);
}

}  // namespace dsa
