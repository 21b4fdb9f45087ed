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
// Design (sm_100a).  Both products are D = X . W per head: 128 batch rows
// are the A operand (M = 128, K-major, 128-byte swizzled) and a slice of the
// head's weight is the B operand (N = up to 256 output features per
// instruction; MN-major: the weight's rows are the K index and its columns
// lie contiguous, loaded by TMA with 128-byte swizzle).  The work is a list of
// (head, feature tile, 128-row tile) items; one persistent CTA per SM walks a
// contiguous run of it.  Warps are specialised (warp 0 TMA, warps 1-4
// producers' helpers, warp 5 one thread issuing tcgen05.mma into tensor-memory
// slots, warps 6-9 the epilogue: a thread reads its row of a slot, 32
// features at a time) and every hand-off is an mbarrier:
//   - the absorbed query keeps a 128 KB weight tile (all 512 features of a
//     head for d_nope = 128) in shared memory across the head's row tiles,
//     loads the bf16 rows by TMA (a 3-D map over [n][H][d_nope]: a box is one
//     64-wide K atom of 128 rows of one head), and writes q_abs through
//     swizzled 64-feature boxes stored by TMA (warps 1-4 copy q_rope through);
//   - the value projection loads the fp32 rows raw by TMA into a ring of
//     stages, which warps 1-4 read into registers (freeing the stage at once)
//     and write, split into two bf16 terms (hi + lo, like the attention
//     weights of the PV product, so the projection keeps near-fp32 inputs),
//     into one of two operand buffers beside the weight slice of that K atom
//     (loaded by TMA from L2); the epilogue stores fp32 rows as 16-byte vectors.
// Every wait is bounded in wall time; a time-out records an error in the
// status block, drains what is in flight, frees tensor memory and returns.
#include <cuda_bf16.h>

#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kWarps = 10;
constexpr int kThreads = 32 * kWarps;
constexpr int kMmaWarp = 5;
constexpr int kTileN = 128;       // batch rows per item
constexpr int kAtomCols = 64;     // weight columns per 128-byte swizzle atom
constexpr int kMaxBoxRows = 256;  // TMA box height limit
constexpr int kAcc = 4;           // tensor-memory accumulators (128 columns each)
constexpr int kMaxStages = 8;
constexpr int kAtomBytes = kTileN * 128;  // one 64-wide K atom of 128 rows, bf16

struct AbsorbParams {
  const float *xf;        // project: o_lat [n, H, K] fp32 (absorb loads q_nope by TMA)
  const uint16_t *rope;   // absorb: q_rope [n, H, P] (nullptr when P == 0)
  uint16_t *out_bf16;     // absorb: q_abs [n, H, M + P]
  float *out_f32;         // project: v_out [n, H, M]
  int n, H, K, M, P;      // rows, heads, reduction length, output features, rope width
  int stages;             // activation stages in shared memory
  int mtile, nchunk;      // features per item (resident weight tile), per accumulator
  int nmt, ntile;         // feature tiles, row tiles
  int vec_out;            // project: v_out is 16-byte aligned (vector stores)
  uint64_t wait_ns;
  DevStatus *status;
};

// shared-memory layout of the absorbed query: [weight tile: mtile / 64 atoms
// x K rows x 128 B][stages: one bf16 K atom of 128 rows][two output boxes per
// epilogue warp][barriers][misc], from a 1024-byte aligned base
constexpr uint32_t kOutBox = 32 * 128;  // 32 rows x 64 bf16 features
struct Layout {
  uint32_t w_bytes, stage_bytes, off_out, off_bars, bytes;
};
__host__ __device__ inline Layout layout_of(int K, int mtile, int stages) {
  Layout l;
  l.w_bytes = static_cast<uint32_t>(mtile / 64 * K * 128);
  l.stage_bytes = kAtomBytes;
  l.off_out = l.w_bytes + static_cast<uint32_t>(stages) * l.stage_bytes;
  l.off_bars = l.off_out + 4u * 2u * kOutBox;
  // full[S], empty[S], tfull[4], tempty[4], wfull, wfree, drain; then misc
  l.bytes = l.off_bars + static_cast<uint32_t>(2 * stages + 2 * kAcc + 3) * 8 + 16;
  return l;
}

// a bounded wait that also gives up once another role has failed
__device__ __forceinline__ bool role_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns,
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

__device__ __forceinline__ void st_shared_u4(uint32_t a, uint32_t x, uint32_t y, uint32_t z,
                                             uint32_t w) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w)
               : "memory");
}

__device__ __forceinline__ uint4 ld_shared_u4(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a)
               : "memory");
  return v;
}

// item u -> (head, feature tile, row tile); heads outermost, row tiles innermost
struct Item {
  int h, mt, t;
};
__device__ __forceinline__ Item item_of(int u, int nmt, int ntile) {
  Item it;
  it.t = u % ntile;
  const int r = u / ntile;
  it.mt = r % nmt;
  it.h = r / nmt;
  return it;
}

// The absorbed query.
__global__ void __launch_bounds__(kThreads, 1)
    absorb_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                  const __grid_constant__ CUtensorMap tmO, const AbsorbParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const int K = p.K, S = p.stages, nkb = K / 64;
  const Layout lay = layout_of(K, p.mtile, S);
  const int NC = p.nchunk, nch = p.mtile / NC, nslot = 32 * 4 * kAcc / NC;
  uint8_t *Ws = smem;                // [mtile / 64 feature atoms][K rows][128 B]
  uint8_t *Xs = smem + lay.w_bytes;  // [S] one bf16 K atom of 128 rows
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + lay.off_bars);
  uint64_t *full = bars, *empty = bars + S;
  uint64_t *tfull = bars + 2 * S, *tempty = tfull + kAcc;
  uint64_t *wfull = tempty + kAcc, *wfree = wfull + 1, *drain = wfree + 1;
  uint32_t *misc = reinterpret_cast<uint32_t *>(drain + 1);  // [0] tmem base, [1] failed
  volatile uint32_t *failed = misc + 1;

  const int tid = threadIdx.x, warp = warp_id(), lane = lane_id();
  const int total = p.H * p.nmt * p.ntile;
  const int u0 = static_cast<int>((static_cast<int64_t>(total) * blockIdx.x) / gridDim.x);
  const int u1 = static_cast<int>((static_cast<int64_t>(total) * (blockIdx.x + 1)) / gridDim.x);
  const uint32_t a_atom = static_cast<uint32_t>(K * 128);

  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < kAcc; ++i) {  // (the first nslot of them)
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);  // one arrive per epilogue warp
    }
    mbar_init(wfull, 1);
    mbar_init(wfree, 1);
    mbar_init(drain, 1);
    misc[1] = 0u;
    fence_barrier_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmO);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&misc[0], 32 * 4 * kAcc);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  // the activations (and, in general, the weights) may come from earlier work
  griddep_wait();
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA
    if (lane == 0) {
      int stage = 0, cur = -1, wgen = 0;
      uint32_t sphase = 0;
      uint32_t armed = 0, armed_par = 0;  // stages with loads in flight, their parity
      bool w_armed = false;               // the last weight load was issued
      bool ok = true;
      uint64_t *land = full;
      for (int u = u0; u < u1 && ok; ++u) {
        const Item it = item_of(u, p.nmt, p.ntile);
        const int wkey = it.h * p.nmt + it.mt;
        if (wkey != cur) {
          // a new weight tile once every product on the old one has completed
          w_armed = false;
          if (wgen > 0 && !role_wait(wfree, static_cast<uint32_t>(wgen - 1) & 1u, p.wait_ns, failed)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(wfull, lay.w_bytes);
          for (int j = 0; j < p.mtile / kAtomCols; ++j)
            for (int r0 = 0; r0 < K; r0 += kMaxBoxRows)
              tma_load_2d(Ws + j * a_atom + r0 * 128, &tmW, it.mt * p.mtile + j * kAtomCols,
                          it.h * K + r0, wfull);
          w_armed = true;
          cur = wkey;
          ++wgen;
        }
        for (int kb = 0; kb < nkb; ++kb) {
          if (!role_wait(&empty[stage], sphase ^ 1u, p.wait_ns, failed)) { ok = false; break; }
          mbar_arrive_expect_tx(&land[stage], lay.stage_bytes);
          tma_load_3d(Xs + stage * lay.stage_bytes, &tmX, kb * 64, it.h, it.t * kTileN, &land[stage]);
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (sphase << stage);
          if (++stage == S) { stage = 0; sphase ^= 1u; }
        }
      }
      if (!ok) {
        // let the loads in flight land before the memory is released
        for (int s = 0; s < S; ++s)
          if (armed & (1u << s)) mbar_wait(&land[s], (armed_par >> s) & 1u, kDrainLimitNs);
        if (w_armed) mbar_wait(wfull, static_cast<uint32_t>(wgen - 1) & 1u, kDrainLimitNs);
      }
    }
  } else if (warp <= 4) {
    const int t4 = tid - 32;  // 0 .. 127
    // ------------------------------------------------------------ rope
    if (p.P > 0) {
      const int pr = p.P / 8;  // 16-byte pieces per row
      for (int u = u0; u < u1; ++u) {
        const Item it = item_of(u, p.nmt, p.ntile);
        if (it.mt != 0) continue;  // the first feature tile's items copy it
        const int b0 = it.t * kTileN, rows = min(kTileN, p.n - b0);
        // eight pieces per thread at a time: all loads in flight before the stores
        for (int pc0 = 0; pc0 < rows * pr; pc0 += 8 * 128) {
          uint4 v[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int pc = pc0 + t4 + 128 * i;
            if (pc < rows * pr) {
              const int r = pc / pr, c = pc - r * pr;
              const int64_t row = static_cast<int64_t>(b0 + r) * p.H + it.h;
              v[i] = __ldg(reinterpret_cast<const uint4 *>(p.rope + row * p.P + c * 8));
            }
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int pc = pc0 + t4 + 128 * i;
            if (pc < rows * pr) {
              const int r = pc / pr, c = pc - r * pr;
              const int64_t row = static_cast<int64_t>(b0 + r) * p.H + it.h;
              *reinterpret_cast<uint4 *>(p.out_bf16 + row * (p.M + p.P) + p.M + c * 8) = v[i];
            }
          }
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    // An item's features go in chunks of NC into tensor-memory slots; with
    // several chunks every K stage of the item stays until its last chunk.
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kTileN, NC, 0, 1);
      const uint32_t ws = smem_u32(Ws), xs = smem_u32(Xs);
      int stage = 0, slot = 0, cur = -1, wgen = 0;
      uint32_t sphase = 0, tphase = 0;
      bool ok = true;
      for (int u = u0; u < u1 && ok; ++u) {
        const Item it = item_of(u, p.nmt, p.ntile);
        const int wkey = it.h * p.nmt + it.mt;
        if (wkey != cur) {
          if (wgen > 0) mma_commit(wfree);  // fires once every product on the old tile is done
          if (!role_wait(wfull, static_cast<uint32_t>(wgen) & 1u, p.wait_ns, failed)) { ok = false; break; }
          cur = wkey;
          ++wgen;
        }
        for (int c = 0; c < nch && ok; ++c) {
          if (!role_wait(&tempty[slot], tphase ^ 1u, p.wait_ns, failed)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d = tmem + static_cast<uint32_t>(slot * NC);
          int st = stage;
          uint32_t sp = sphase;
          for (int kb = 0; kb < nkb; ++kb) {
            if (!role_wait(&full[st], sp, p.wait_ns, failed)) { ok = false; break; }
            tc_fence_after();
            const uint32_t xb = xs + static_cast<uint32_t>(st) * lay.stage_bytes;
            const uint32_t wb = ws + static_cast<uint32_t>(c * NC / kAtomCols) * a_atom;
            for (int ks = 0; ks < 4; ++ks)
              mma_bf16(d, smem_desc(xb + ks * 32, 16, 1024, kLayoutSW128),
                       smem_desc(wb + (kb * 4 + ks) * 2048, a_atom, 1024, kLayoutSW128), idesc,
                       (kb | ks) != 0 ? 1u : 0u);
            if (c == nch - 1) mma_commit(&empty[st]);  // the stage's last use
            if (++st == S) { st = 0; sp ^= 1u; }
          }
          if (!ok) break;
          mma_commit(&tfull[slot]);
          if (++slot == nslot) { slot = 0; tphase ^= 1u; }
          if (c == nch - 1) { stage = st; sphase = sp; }
        }
      }
      if (*failed) {
        mma_commit(drain);  // fires once every product issued above has completed
        mbar_wait(drain, 0u, kDrainLimitNs);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // tensor-memory lane quadrant: rows 32 q ..
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    // (the absorbed query) this warp's two output boxes
    const uint32_t obox = smem_u32(smem + lay.off_out) + static_cast<uint32_t>(warp - 6) * 2u * kOutBox;
    int ob = 0;
    int slot = 0;
    uint32_t tphase = 0;
    bool ok = true;
    for (int u = u0; u < u1 && ok; ++u) {
      const Item it = item_of(u, p.nmt, p.ntile);
      for (int c = 0; c < nch; ++c) {
        bool okw = true;
        if (lane == 0) okw = role_wait(&tfull[slot], tphase, p.wait_ns, failed);
        if (!__shfl_sync(0xffffffffu, okw, 0)) { ok = false; break; }
        tc_fence_after();
        const int fc = it.mt * p.mtile + c * NC;  // the chunk's first feature
        {
          // 64 features of the warp's 32 rows at a time, rounded to bf16 into
          // one of the warp's two swizzled boxes, which lane 0 stores by TMA
          // (rows past n are clipped); a box is rewritten once its previous
          // store has been read
          for (int c0 = 0; c0 < NC && fc + c0 < p.M; c0 += 64) {
            uint32_t h2[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              uint32_t v[32];
              tmem_ld_32x32b_x32(tmem + lane_off + static_cast<uint32_t>(slot * NC + c0 + 32 * half), v);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const __nv_bfloat162 t = __floats2bfloat162_rn(__uint_as_float(v[2 * j]),
                                                               __uint_as_float(v[2 * j + 1]));
                h2[16 * half + j] = *reinterpret_cast<const uint32_t *>(&t);
              }
            }
            if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
            __syncwarp();
            const uint32_t box = obox + static_cast<uint32_t>(ob) * kOutBox;
#pragma unroll
            for (int j = 0; j < 8; ++j)
              st_shared_u4(box + lane * 128 + ((j ^ (lane & 7)) << 4), h2[4 * j], h2[4 * j + 1],
                           h2[4 * j + 2], h2[4 * j + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(&tmO, box, fc + c0, it.h, it.t * kTileN + 32 * q);
              asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            }
            ob ^= 1;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[slot]);
        if (++slot == nslot) { slot = 0; tphase ^= 1u; }
      }
    }
    // the boxes' stores complete before the kernel ends
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == 0 && *failed) report(p.status, kErrTimeout, (kKernAbsorb << 24) | 1u);
  if (warp == kMmaWarp) {
    __syncwarp();
    tmem_dealloc(tmem, 32 * 4 * kAcc);
  }
}

// The value projection, whose fp32 rows cannot be the MMA operand as they
// land: warp 0 loads them raw (lane 0: fp32 stages by TMA) and the weight
// slice of each K atom (lane 1: MN-major, by TMA) into an operand buffer;
// warps 1-4 read a raw stage into registers (freeing it at once, so that
// several stay in flight), split each value into hi + lo bf16 terms and
// write them, swizzled, beside the weight slice; warp 5 issues the MMAs of
// an item's K atoms (features in chunks of NC, one tensor-memory slot each);
// warps 6-9 store rows of the accumulators.  (The rows' TMA boxes are 128
// rows of 256 bytes: the copies alone run at about 28 GB/s per SM, which
// bounds this kernel below the HBM rate.)
constexpr int kOps = 2;        // operand buffers
constexpr int kMaxSlots = 8;   // tensor-memory slots (512 columns / NC)
struct ProjLayout {
  uint32_t raw_bytes, op_bytes, off_op, off_bars, bytes;
};
__host__ __device__ inline ProjLayout proj_layout(int mtile, int raws) {
  ProjLayout l;
  l.raw_bytes = 2 * kAtomBytes;                                  // 128 rows x 64 fp32
  l.op_bytes = 2 * kAtomBytes + static_cast<uint32_t>(mtile) * 128;  // hi, lo, weight slice
  l.off_op = static_cast<uint32_t>(raws) * l.raw_bytes;
  l.off_bars = l.off_op + kOps * l.op_bytes;
  // raw_full[R], raw_empty[R], op_full[2], op_empty[2], tfull[8], tempty[8], drain; misc
  l.bytes = l.off_bars + static_cast<uint32_t>(2 * raws + 2 * kOps + 2 * kMaxSlots + 1) * 8 + 16;
  return l;
}

__global__ void __launch_bounds__(kThreads, 1)
    project_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                   const AbsorbParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const int K = p.K, R = p.stages, nkb = K / 64, MT = p.mtile;
  const int NC = p.nchunk, nch = MT / NC, nslot = 32 * 4 * kAcc / NC;
  const ProjLayout lay = proj_layout(MT, R);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + lay.off_bars);
  uint64_t *raw_full = bars, *raw_empty = bars + R;
  uint64_t *op_full = bars + 2 * R, *op_empty = op_full + kOps;
  uint64_t *tfull = op_empty + kOps, *tempty = tfull + kMaxSlots, *drain = tempty + kMaxSlots;
  uint32_t *misc = reinterpret_cast<uint32_t *>(drain + 1);  // [0] tmem base, [1] failed
  volatile uint32_t *failed = misc + 1;
  auto raw_at = [&](int r) { return smem + static_cast<uint32_t>(r) * lay.raw_bytes; };
  auto op_at = [&](int o) { return smem + lay.off_op + static_cast<uint32_t>(o) * lay.op_bytes; };

  const int tid = threadIdx.x, warp = warp_id(), lane = lane_id();
  const int total = p.H * p.nmt * p.ntile;
  const int u0 = static_cast<int>((static_cast<int64_t>(total) * blockIdx.x) / gridDim.x);
  const int u1 = static_cast<int>((static_cast<int64_t>(total) * (blockIdx.x + 1)) / gridDim.x);

  if (tid == 0) {
    for (int i = 0; i < R; ++i) {
      mbar_init(&raw_full[i], 1);
      mbar_init(&raw_empty[i], 4);  // one arrive per converting warp
    }
    for (int i = 0; i < kOps; ++i) {
      mbar_init(&op_full[i], 5);  // the weight slice's TMA and the four converting warps
      mbar_init(&op_empty[i], 1);
    }
    for (int i = 0; i < kMaxSlots; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);  // one arrive per epilogue warp
    }
    mbar_init(drain, 1);
    misc[1] = 0u;
    fence_barrier_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&misc[0], 32 * 4 * kAcc);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  griddep_wait();
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA
    if (lane < 2) {
      const int n_ring = lane == 0 ? R : kOps;
      uint64_t *fullb = lane == 0 ? raw_full : op_full;
      uint64_t *emptyb = lane == 0 ? raw_empty : op_empty;
      int idx = 0;
      uint32_t ph = 0;
      uint32_t armed = 0, armed_par = 0;
      for (int u = u0; u < u1; ++u) {
        const Item it = item_of(u, p.nmt, p.ntile);
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!role_wait(&emptyb[idx], ph ^ 1u, p.wait_ns, failed)) { ok = false; break; }
          if (lane == 0) {
            mbar_arrive_expect_tx(&fullb[idx], lay.raw_bytes);
            tma_load_3d(raw_at(idx), &tmX, kb * 64, it.h, it.t * kTileN, &fullb[idx]);
          } else {
            mbar_arrive_expect_tx(&fullb[idx], static_cast<uint32_t>(MT) * 128);
            uint8_t *wdst = op_at(idx) + 2 * kAtomBytes;
            for (int j = 0; j < MT / kAtomCols; ++j)
              tma_load_2d(wdst + j * (64 * 128), &tmW, it.mt * MT + j * kAtomCols, it.h * K + kb * 64,
                          &fullb[idx]);
          }
          armed |= 1u << idx;
          armed_par = (armed_par & ~(1u << idx)) | (ph << idx);
          if (++idx == n_ring) { idx = 0; ph ^= 1u; }
        }
        if (!ok) break;
      }
      if (*failed) {
        // let the loads in flight land before the memory is released (an
        // operand buffer's phase also needs the converters, so wait with a
        // bound either way)
        for (int s = 0; s < n_ring; ++s)
          if (armed & (1u << s)) mbar_wait(&fullb[s], (armed_par >> s) & 1u, kDrainLimitNs / 8);
      }
    }
  } else if (warp <= 4) {
    // ------------------------------------------------------------ hi + lo
    const int t4 = tid - 32;  // 0 .. 127
    int r = 0, o = 0;
    uint32_t rph = 0, oph = 0;
    bool ok = true;
    for (int u = u0; u < u1 && ok; ++u) {
      for (int kb = 0; kb < nkb; ++kb) {
        bool okw = true;
        if (lane == 0) okw = role_wait(&raw_full[r], rph, p.wait_ns, failed);
        if (!__shfl_sync(0xffffffffu, okw, 0)) { ok = false; break; }
        const uint32_t rb = smem_u32(raw_at(r));
        uint4 x[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int q = t4 + 128 * i, rr = q >> 3, c = q & 7;
          x[2 * i] = ld_shared_u4(rb + rr * 256 + c * 32);
          x[2 * i + 1] = ld_shared_u4(rb + rr * 256 + c * 32 + 16);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&raw_empty[r]);  // this warp's reads are done
        if (++r == R) { r = 0; rph ^= 1u; }
        if (lane == 0) okw = role_wait(&op_empty[o], oph ^ 1u, p.wait_ns, failed);
        if (!__shfl_sync(0xffffffffu, okw, 0)) { ok = false; break; }
        const uint32_t ob = smem_u32(op_at(o));
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int q = t4 + 128 * i, rr = q >> 3, c = q & 7;
          const uint32_t w8[8] = {x[2 * i].x, x[2 * i].y, x[2 * i].z, x[2 * i].w,
                                  x[2 * i + 1].x, x[2 * i + 1].y, x[2 * i + 1].z, x[2 * i + 1].w};
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float v0 = __uint_as_float(w8[2 * j]), v1 = __uint_as_float(w8[2 * j + 1]);
            const __nv_bfloat162 a = __floats2bfloat162_rn(v0, v1);
            const __nv_bfloat162 e = __floats2bfloat162_rn(v0 - __low2float(a), v1 - __high2float(a));
            hi[j] = *reinterpret_cast<const uint32_t *>(&a);
            lo[j] = *reinterpret_cast<const uint32_t *>(&e);
          }
          const uint32_t off = static_cast<uint32_t>(rr * 128 + ((c ^ (rr & 7)) << 4));
          st_shared_u4(ob + off, hi[0], hi[1], hi[2], hi[3]);
          st_shared_u4(ob + kAtomBytes + off, lo[0], lo[1], lo[2], lo[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&op_full[o]);
        if (++o == kOps) { o = 0; oph ^= 1u; }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kTileN, NC, 0, 1);
      int slot = 0, o = 0;
      uint32_t tph = 0, oph = 0;
      bool ok = true;
      for (int u = u0; u < u1 && ok; ++u) {
        // the item's chunks take the next nch slots
        int s0 = slot;
        for (int c = 0; c < nch && ok; ++c) {
          if (!role_wait(&tempty[slot], tph ^ 1u, p.wait_ns, failed)) ok = false;
          if (++slot == nslot) { slot = 0; tph ^= 1u; }
        }
        if (!ok) break;
        tc_fence_after();
        for (int kb = 0; kb < nkb; ++kb) {
          if (!role_wait(&op_full[o], oph, p.wait_ns, failed)) { ok = false; break; }
          tc_fence_after();
          const uint32_t ob = smem_u32(op_at(o));
          for (int c = 0; c < nch; ++c) {
            const uint32_t d = tmem + static_cast<uint32_t>(((s0 + c) % nslot) * NC);
            const uint32_t wb = ob + 2 * kAtomBytes + static_cast<uint32_t>(c * NC / kAtomCols) * (64 * 128);
            for (int term = 0; term < 2; ++term)
              for (int ks = 0; ks < 4; ++ks)
                mma_bf16(d, smem_desc(ob + term * kAtomBytes + ks * 32, 16, 1024, kLayoutSW128),
                         smem_desc(wb + ks * 2048, 64 * 128, 1024, kLayoutSW128), idesc,
                         (kb | term | ks) != 0 ? 1u : 0u);
          }
          mma_commit(&op_empty[o]);
          if (++o == kOps) { o = 0; oph ^= 1u; }
        }
        if (!ok) break;
        for (int c = 0; c < nch; ++c) mma_commit(&tfull[(s0 + c) % nslot]);
      }
      if (*failed) {
        mma_commit(drain);  // fires once every product issued above has completed
        mbar_wait(drain, 0u, kDrainLimitNs);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // tensor-memory lane quadrant: rows 32 q ..
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    int slot = 0;
    uint32_t tph = 0;
    bool ok = true;
    for (int u = u0; u < u1 && ok; ++u) {
      const Item it = item_of(u, p.nmt, p.ntile);
      const int b = it.t * kTileN + 32 * q + lane;  // this thread's row
      const int64_t row = static_cast<int64_t>(b) * p.H + it.h;
      for (int c = 0; c < nch; ++c) {
        bool okw = true;
        if (lane == 0) okw = role_wait(&tfull[slot], tph, p.wait_ns, failed);
        if (!__shfl_sync(0xffffffffu, okw, 0)) { ok = false; break; }
        tc_fence_after();
        const int fc = it.mt * MT + c * NC;
        for (int c0 = 0; c0 < NC && fc + c0 < p.M; c0 += 32) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tmem + lane_off + static_cast<uint32_t>(slot * NC + c0), v);
          tmem_ld_wait();
          if (b < p.n) {
            float *dst = p.out_f32 + row * p.M + fc + c0;
            if (p.vec_out) {
#pragma unroll
              for (int j = 0; j < 8; ++j)
                reinterpret_cast<uint4 *>(dst)[j] =
                    make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) dst[j] = __uint_as_float(v[j]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[slot]);
        if (++slot == nslot) { slot = 0; tph ^= 1u; }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == 0 && *failed) report(p.status, kErrTimeout, (kKernAbsorb << 24) | 2u);
  if (warp == kMmaWarp) {
    __syncwarp();
    tmem_dealloc(tmem, 32 * 4 * kAcc);
  }
}

dsa_status_t launch_project(const AbsorbLaunch &a, cudaStream_t stream) {
  const int K = a.K;
  const size_t optin = device_max_smem_optin();
  // features per item: up to 256 (a head's, for d_v <= 256), in chunks of up to 256
  const int mtile = std::min(a.M, 256);
  const int nchunk = mtile % 256 == 0 ? 256 : (mtile % 128 == 0 ? 128 : 64);
  int raws = 6;
  while (raws > 2 && 1024 + proj_layout(mtile, raws).bytes > optin) --raws;
  const size_t smem = std::max<size_t>(1024 + proj_layout(mtile, raws).bytes, optin / 2 + 1024);
  if (smem > optin) return DSA_ERR_UNSUPPORTED;
  if (func_attr_once(reinterpret_cast<const void *>(project_kernel),
                     cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(optin)) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  CUtensorMap tmW, tmX;
  // the weights as [H * K rows][M columns], one K atom (64 rows) of 64 columns per box
  if (!make_map_2d(&tmW, a.w, static_cast<uint64_t>(a.M), static_cast<uint64_t>(a.H) * K, 64, 64, 128))
    return DSA_ERR_CUDA;
  // the fp32 rows as [n][H][K]: a box is one 64-wide K atom of 128 rows of one head
  if (!make_map_3d(&tmX, a.xf, 4, static_cast<uint64_t>(K), static_cast<uint64_t>(a.H),
                   static_cast<uint64_t>(a.n), static_cast<uint64_t>(K) * 4,
                   static_cast<uint64_t>(a.H) * K * 4, 64, 1, kTileN, false))
    return DSA_ERR_CUDA;
  AbsorbParams p = {};
  p.xf = a.xf;
  p.out_f32 = a.out_f32;
  p.n = a.n;
  p.H = a.H;
  p.K = K;
  p.M = a.M;
  p.P = 0;
  p.stages = raws;
  p.mtile = mtile;
  p.nchunk = nchunk;
  p.vec_out = (reinterpret_cast<uintptr_t>(a.out_f32) & 15u) == 0 ? 1 : 0;
  p.nmt = (a.M + mtile - 1) / mtile;
  p.ntile = (a.n + kTileN - 1) / kTileN;
  p.wait_ns = wait_limit_ns();
  p.status = a.status;
  const int64_t items = static_cast<int64_t>(a.H) * p.nmt * p.ntile;
  if (items > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  const int grid = static_cast<int>(std::min<int64_t>(items, device_sm_count()));
  if (launch_pdl(project_kernel, dim3(grid), dim3(kThreads), smem, stream, 1, tmW, tmX, p) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

dsa_status_t launch_absorb_query(const AbsorbLaunch &a, cudaStream_t stream) {
  const int K = a.K, nkb = K / 64;
  const size_t optin = device_max_smem_optin();
  // the features of an item: as many as a 128 KB weight tile holds (all of a
  // head's when they fit), in accumulator chunks of up to 256
  int mtile = std::min(a.M, std::min(512, (131072 / (2 * K)) / 64 * 64));
  auto chunk_of = [](int mt) { return mt % 256 == 0 ? 256 : (mt % 128 == 0 ? 128 : 64); };
  // as many activation stages as shared memory holds beside the weight tile
  // and the output boxes (at least two); the kernel owns its SM (one CTA: all
  // of tensor memory)
  auto stages_for = [&](int mt) {
    int st = kMaxStages;
    while (st > 2 && 1024 + layout_of(K, mt, st).bytes > optin) --st;
    return st;
  };
  int stages = stages_for(mtile);
  // several chunks per item keep every K stage of the item until the last one
  if (mtile / chunk_of(mtile) > 1 && stages < nkb) {
    mtile = chunk_of(mtile);
    stages = stages_for(mtile);
  }
  const size_t smem = std::max<size_t>(1024 + layout_of(K, mtile, stages).bytes, optin / 2 + 1024);
  if (smem > optin) return DSA_ERR_UNSUPPORTED;
  if (func_attr_once(reinterpret_cast<const void *>(absorb_kernel),
                     cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(optin)) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  CUtensorMap tmW, tmX, tmO;
  // the weights as [H * K rows][M columns]; boxes of 64 columns x min(K, 256) rows
  if (!make_map_2d(&tmW, a.w, static_cast<uint64_t>(a.M), static_cast<uint64_t>(a.H) * K, 64,
                   std::min(K, kMaxBoxRows), 128))
    return DSA_ERR_CUDA;
  // the rows as [n][H][K]: a box is one 64-wide K atom of 128 rows of one head
  if (!make_map_3d(&tmX, a.x, 2, static_cast<uint64_t>(K), static_cast<uint64_t>(a.H),
                   static_cast<uint64_t>(a.n), static_cast<uint64_t>(K) * 2,
                   static_cast<uint64_t>(a.H) * K * 2, 64, 1, kTileN, true))
    return DSA_ERR_CUDA;
  // the output as [n][H][M + P]: boxes of 64 features x 32 rows
  if (!make_map_3d(&tmO, a.out_bf16, 2, static_cast<uint64_t>(a.M + a.P), static_cast<uint64_t>(a.H),
                   static_cast<uint64_t>(a.n), static_cast<uint64_t>(a.M + a.P) * 2,
                   static_cast<uint64_t>(a.H) * (a.M + a.P) * 2, 64, 1, 32, true))
    return DSA_ERR_CUDA;
  AbsorbParams p = {};
  p.rope = a.rope;
  p.out_bf16 = a.out_bf16;
  p.n = a.n;
  p.H = a.H;
  p.K = K;
  p.M = a.M;
  p.P = a.P;
  p.stages = stages;
  p.mtile = mtile;
  p.nchunk = chunk_of(mtile);
  p.nmt = (a.M + mtile - 1) / mtile;
  p.ntile = (a.n + kTileN - 1) / kTileN;
  p.wait_ns = wait_limit_ns();
  p.status = a.status;
  const int64_t items = static_cast<int64_t>(a.H) * p.nmt * p.ntile;
  if (items > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  const int grid = static_cast<int>(std::min<int64_t>(items, device_sm_count()));
  if (launch_pdl(absorb_kernel, dim3(grid), dim3(kThreads), smem, stream, 1, tmW, tmX, tmO, p) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

}  // namespace

dsa_status_t launch_absorb(const AbsorbLaunch &a, cudaStream_t stream) {
  return a.project ? launch_project(a, stream) : launch_absorb_query(a, stream);
}

}  // namespace dsa
