// The C ABI of libdsa: argument checks on the host, workspace layout, and the
// launch sequence of each entry point.  See include/dsa.h for the contract.
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include <cudaTypedefs.h>

#include "dsa_internal.h"

namespace dsa {

uint64_t wait_limit_ns() {
  static const uint64_t v = [] {
    const char *s = getenv("DSA_WAIT_LIMIT_NS");
    if (s != nullptr && *s != '\0') return static_cast<uint64_t>(strtoull(s, nullptr, 10));
    return static_cast<uint64_t>(1000000000ull);
  }();
  return v;
}

int debug_stall() {
  static const int v = [] {
    const char *s = getenv("DSA_DEBUG_STALL");
    return (s != nullptr && *s != '\0') ? atoi(s) : 0;
  }();
  return v;
}

namespace {
constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices];
size_t g_smem_optin[kMaxDevices];

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return -1;
  return d;
}
}  // namespace

int device_sm_count() {
  const int d = current_device();
  if (d < 0) return 148;
  if (g_sm_count[d] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || v <= 0)
      return 148;
    g_sm_count[d] = v;
  }
  return g_sm_count[d];
}

size_t device_max_smem_optin() {
  const int d = current_device();
  if (d < 0) return 232448;
  if (g_smem_optin[d] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, d) != cudaSuccess ||
        v <= 0)
      return 232448;
    g_smem_optin[d] = static_cast<size_t>(v);
  }
  return g_smem_optin[d];
}

namespace {
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
  }();
  return fn;
}
}  // namespace

bool make_map_2d(CUtensorMap *map, const void *base, uint64_t cols, uint64_t rows,
                 uint32_t box_cols, uint32_t box_rows, int aw) {
  auto encode = get_encode_fn();
  if (encode == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      aw == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// [d2][d1][d0] elements of `esize` bytes (2: bf16, 4: fp32) with row strides
// s1 and s2 bytes, boxes of b0 x b1 x b2 elements; 128-byte swizzle (b0 *
// esize must then be 128) or none
bool make_map_3d(CUtensorMap *map, const void *base, int esize, uint64_t d0, uint64_t d1,
                 uint64_t d2, uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2,
                 bool swizzle) {
  auto encode = get_encode_fn();
  if (encode == nullptr || (esize != 2 && esize != 4)) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = encode(map, esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                      3, const_cast<void *>(base), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE,
                      swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// bytes (the FP8 index keys and query terms); aw = swizzle width, 128 or 64
bool make_map_2d_u8(CUtensorMap *map, const void *base, uint64_t cols, uint64_t rows,
                    uint32_t box_cols, uint32_t box_rows, int aw) {
  auto encode = get_encode_fn();
  if (encode == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      aw == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

size_t device_smem_per_sm() {
  static size_t cached[kMaxDevices];
  const int d = current_device();
  if (d < 0) return 233472;
  if (cached[d] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerMultiprocessor, d) != cudaSuccess ||
        v <= 0)
      return 233472;
    cached[d] = static_cast<size_t>(v);
  }
  return cached[d];
}

namespace {
thread_local char g_last_error[256];
}  // namespace

cudaError_t note_cuda_error(cudaError_t err, const char *where) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%d)", where, cudaGetErrorString(err),
           static_cast<int>(err));
  return err;
}

cudaError_t func_attr_once(const void *kernel, cudaFuncAttribute attr, int value) {
  struct Entry {
    int dev;
    const void *kernel;
    cudaFuncAttribute attr;
    int value;
  };
  static std::mutex mu;
  static std::vector<Entry> done;
  const int d = current_device();
  std::lock_guard<std::mutex> lock(mu);
  // one entry per (device, kernel, attribute) holding the value last set: a
  // kernel has one value per attribute, so a new value is set again
  Entry *slot = nullptr;
  for (Entry &e : done)
    if (e.dev == d && e.kernel == kernel && e.attr == attr) slot = &e;
  if (slot != nullptr && slot->value == value) return cudaSuccess;
  const cudaError_t err = cudaFuncSetAttribute(kernel, attr, value);
  if (err != cudaSuccess) {
    if (slot != nullptr) slot->value = INT32_MIN;  // unknown now: set again next time
    return note_cuda_error(err, "cudaFuncSetAttribute");
  }
  if (slot != nullptr) slot->value = value;
  else if (d >= 0) done.push_back(Entry{d, kernel, attr, value});
  return err;
}

namespace {

constexpr size_t kStatusBytes = sizeof(DevStatus);
static_assert(kStatusBytes == DSA_STATUS_WORKSPACE_BYTES, "status block size in the header");

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
cudaStream_t as_stream(dsa_stream_t s) {
  return s ? reinterpret_cast<cudaStream_t>(s) : cudaStreamPerThread;
}

// tokens the longest query row sees
int64_t max_keys(const dsa_dims_t &d, const dsa_cache_t &c) {
  return d.causal ? static_cast<int64_t>(d.q_pos0) + d.n_q : static_cast<int64_t>(c.max_seq_len);
}
int64_t scores_ld(const dsa_dims_t &d, const dsa_cache_t &c) {
  return std::max<int64_t>(4, (max_keys(d, c) + 3) & ~static_cast<int64_t>(3));
}

}  // namespace

dsa_status_t check_dims_common(const dsa_dims_t *d) {
  if (d == nullptr) return DSA_ERR_INVALID_ARG;
  if (d->n_q < 0 || d->causal < 0 || d->causal > 1 || d->q_pos0 < 0) return DSA_ERR_INVALID_ARG;
  if (d->causal == 0 && d->q_pos0 != 0) return DSA_ERR_INVALID_ARG;
  return DSA_OK;
}

dsa_status_t check_cache(const dsa_cache_t *c, const dsa_dims_t &d) {
  if (c == nullptr) return DSA_ERR_INVALID_ARG;
  if (c->seq_lens == nullptr || c->block_table == nullptr) return DSA_ERR_INVALID_ARG;
  if (!aligned4(c->seq_lens) || !aligned4(c->block_table)) return DSA_ERR_INVALID_ARG;
  if (c->page_size != kPageSize) return DSA_ERR_UNSUPPORTED;
  if (c->num_seqs < 1 || c->max_pages < 1 || c->num_pages < 1) return DSA_ERR_INVALID_ARG;
  if (c->max_seq_len < 0) return DSA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(c->max_seq_len) > static_cast<int64_t>(c->max_pages) * kPageSize)
    return DSA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(c->num_pages) * kPageSize > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  if (d.causal == 0) {
    if (c->num_seqs != d.n_q) return DSA_ERR_INVALID_ARG;
  } else {
    if (static_cast<int64_t>(d.q_pos0) + d.n_q > static_cast<int64_t>(c->max_pages) * kPageSize)
      return DSA_ERR_INVALID_ARG;
  }
  return DSA_OK;
}

dsa_status_t check_mla_dims(const dsa_dims_t &d) {
  if (d.topk < 1 || d.topk > 65536) return DSA_ERR_UNSUPPORTED;
  if (d.H < 1 || d.H > 64) return DSA_ERR_UNSUPPORTED;
  if (d.R < 64 || d.R > 512 || d.R % 64 != 0) return DSA_ERR_UNSUPPORTED;
  if (d.P < 0 || d.P % 16 != 0 || d.R + d.P > 576) return DSA_ERR_UNSUPPORTED;
  if (!isfinite(d.scale)) return DSA_ERR_INVALID_ARG;
  if (d.n_q > 65535) return DSA_ERR_UNSUPPORTED;  // grid.y
  return DSA_OK;
}

namespace {

dsa_status_t check_indexer_dims(const dsa_dims_t &d) {
  if (d.H_I < 1 || d.H_I > 64) return DSA_ERR_UNSUPPORTED;
  if (d.D_I != 32 && d.D_I != 64 && d.D_I != 128) return DSA_ERR_UNSUPPORTED;
  // the indexer walks row groups out of a shared-memory table
  const int64_t groups = d.causal ? (d.n_q + 3) / 4 : d.n_q;
  if (groups > 8192) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

DevStatus *status_of(void *ws) { return static_cast<DevStatus *>(ws); }

dsa_status_t check_ws(void *ws, size_t ws_bytes, size_t need) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return DSA_ERR_WORKSPACE;
  if (ws_bytes < need) return DSA_ERR_WORKSPACE;
  return DSA_OK;
}

#define DSA_TRY(expr)                        \
  do {                                       \
    const dsa_status_t st__ = (expr);        \
    if (st__ != DSA_OK) return st__;         \
  } while (0)

// FP8-key indexer region after the status block: the E4M3 query terms
// [2][n_q][H_I][D_I] bytes, then the scaled head weights [n_q][H_I] fp32
size_t k8_q_bytes(const dsa_dims_t &d) {
  return align256(2 * static_cast<size_t>(d.n_q) * d.H_I * d.D_I);
}
size_t k8_region_bytes(const dsa_dims_t &d) {
  return k8_q_bytes(d) + align256(static_cast<size_t>(d.n_q) * d.H_I * 4);
}

// device staging of dsa_attention_forward_host, after the step's workspace:
// q_idx, w, q, seq_lens, block_table, then idx, out, lse, each 256-aligned
struct HostStage {
  size_t q_idx, w, q, seq_lens, block_table, idx, out, lse;
};
HostStage host_stage_sizes(const dsa_dims_t &d, const dsa_cache_t &c) {
  const size_t n = static_cast<size_t>(d.n_q);
  HostStage h;
  h.q_idx = n * d.H_I * d.D_I * 2;
  h.w = n * d.H_I * 4;
  h.q = n * d.H * (d.R + d.P) * 2;
  h.seq_lens = static_cast<size_t>(c.num_seqs) * 4;
  h.block_table = static_cast<size_t>(c.num_seqs) * c.max_pages * 4;
  h.idx = n * d.topk * 4;
  h.out = n * d.H * d.R * 4;
  h.lse = n * d.H * 4;
  return h;
}
// the device address of a pinned, mapped host buffer, or nullptr for memory
// the device cannot address (pageable host memory, or not host memory at all)
void *mapped_host(const void *p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return (at.type == cudaMemoryTypeHost) ? at.devicePointer : nullptr;
}

size_t host_stage_bytes(const dsa_dims_t &d, const dsa_cache_t &c) {
  const HostStage h = host_stage_sizes(d, c);
  return align256(h.q_idx) + align256(h.w) + align256(h.q) + align256(h.seq_lens) +
         align256(h.block_table) + align256(h.idx) + align256(h.out) + align256(h.lse);
}

size_t ws_bytes_for(dsa_op_t op, const dsa_dims_t &d, const dsa_cache_t &c) {
  switch (op) {
    case DSA_OP_INDEXER_SCORES:
    case DSA_OP_TOPK:
    case DSA_OP_CACHE_APPEND:
      return kStatusBytes;
    case DSA_OP_INDEXER_SCORES_K8:
      return kStatusBytes + k8_region_bytes(d);
    case DSA_OP_ATTENTION_FORWARD_K8:
    case DSA_OP_ATTENTION_FORWARD_FP8:
      return k8_region_bytes(d) + ws_bytes_for(DSA_OP_ATTENTION_FORWARD, d, c);
    case DSA_OP_SPARSE_MLA_DECODE:
    case DSA_OP_SPARSE_MLA_PREFILL:
      return kStatusBytes + align256(mla_scratch_bytes(d.n_q, d.topk, d.R));
    case DSA_OP_ATTENTION_FORWARD: {
      const size_t scores = static_cast<size_t>(d.n_q) * scores_ld(d, c) * 4;
      const size_t idx = static_cast<size_t>(d.n_q) * d.topk * 4;
      return kStatusBytes + align256(scores) + align256(idx) +
             align256(mla_scratch_bytes(d.n_q, d.topk, d.R));
    }
    case DSA_OP_ATTENTION_FORWARD_HOST:
      return ws_bytes_for(DSA_OP_ATTENTION_FORWARD, d, c) + host_stage_bytes(d, c);
  }
  return 0;
}

// k8_pages != nullptr: E4M3 index keys with one fp32 scale per key row
// (k_scale); k8_region (k8_region_bytes) receives the E4M3 query terms and the
// scaled head weights
dsa_status_t run_indexer(const uint16_t *q_idx, const float *w, const uint16_t *k_pages,
                         const dsa_cache_t &c, const dsa_dims_t &d, float *scores, int64_t ld,
                         DevStatus *st, cudaStream_t s, const uint8_t *k8_pages = nullptr,
                         const float *k_scale = nullptr, uint8_t *k8_region = nullptr,
                         const void *aux_src = nullptr, void *aux_dst = nullptr,
                         size_t aux_bytes = 0) {
  IndexerLaunch a;
  a.q_idx = q_idx;
  a.w = w;
  a.k_pages = k_pages;
  a.k8_pages = k8_pages;
  a.k_scale = k_scale;
  if (k8_pages != nullptr) {
    uint8_t *q8 = k8_region;
    float *w8 = reinterpret_cast<float *>(k8_region + k8_q_bytes(d));
    DSA_TRY(launch_q8_prep(q_idx, w, q8, w8, d.n_q, d.H_I, d.D_I, s));
    a.q8 = q8;
    a.w = w8;
  }
  a.seq_lens = c.seq_lens;
  a.block_table = c.block_table;
  a.scores = scores;
  a.ld = ld;
  a.n_q = d.n_q;
  a.H_I = d.H_I;
  a.D_I = d.D_I;
  a.causal = d.causal;
  a.q_pos0 = d.q_pos0;
  a.num_seqs = c.num_seqs;
  a.max_pages = c.max_pages;
  a.num_pages = c.num_pages;
  a.max_seq_len = c.max_seq_len;
  a.status = st;
  a.aux_src = aux_src;
  a.aux_dst = aux_dst;
  a.aux_bytes = aux_bytes;
  return launch_indexer(a, s);
}

dsa_status_t run_topk(const float *scores, int64_t ld, int n_q, const int32_t *valid_len,
                      int causal_base, int k, int32_t *idx, int max_len, DevStatus *st,
                      cudaStream_t s) {
  TopkLaunch a;
  a.scores = scores;
  a.ld = ld;
  a.n_q = n_q;
  a.valid_len = valid_len;
  a.causal_base = causal_base;
  a.k = k;
  a.idx = idx;
  a.max_len = max_len;
  a.status = st;
  return launch_topk(a, s);
}

// latent8 != nullptr: E4M3 latent rows with one fp32 scale per row (lat_scale)
dsa_status_t run_mla(const uint16_t *q, const uint16_t *latent, const dsa_cache_t &c,
                     const int32_t *idx, const dsa_dims_t &d, float *out, float *lse, void *scratch,
                     size_t scratch_bytes, DevStatus *st, cudaStream_t s, int early_q = 0,
                     const uint8_t *latent8 = nullptr, const float *lat_scale = nullptr) {
  MlaLaunch a;
  a.early_q = early_q;
  a.q = q;
  a.latent = latent;
  a.latent8 = latent8;
  a.lat_scale = lat_scale;
  a.idx = idx;
  a.seq_lens = c.seq_lens;
  a.block_table = c.block_table;
  a.out = out;
  a.lse = lse;
  a.n_q = d.n_q;
  a.H = d.H;
  a.R = d.R;
  a.P = d.P;
  a.topk = d.topk;
  a.causal = d.causal;
  a.q_pos0 = d.q_pos0;
  a.max_pages = c.max_pages;
  a.num_pages = c.num_pages;
  a.scale = d.scale;
  a.scratch = scratch;
  a.scratch_bytes = scratch_bytes;
  a.status = st;
  return launch_mla(a, s);
}

// the sparse MLA entry for bf16 latent rows (latent_pages) or E4M3 rows
// (latent8_pages + lat_scale)
dsa_status_t mla_entry(const uint16_t *q, const uint16_t *latent_pages, const uint8_t *latent8_pages,
                       const float *lat_scale, const dsa_cache_t *cache, const int32_t *idx,
                       const dsa_dims_t *dims, float *out, float *lse, void *ws, size_t ws_bytes,
                       dsa_stream_t stream, int want_causal) {
  DSA_TRY(check_dims_common(dims));
  if (dims->causal != want_causal) return DSA_ERR_INVALID_ARG;
  DSA_TRY(check_mla_dims(*dims));
  DSA_TRY(check_cache(cache, *dims));
  const void *lat = latent8_pages ? static_cast<const void *>(latent8_pages) : latent_pages;
  if (q == nullptr || lat == nullptr || idx == nullptr || out == nullptr || lse == nullptr)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(lat) || !aligned4(idx) || !aligned4(out) || !aligned4(lse) ||
      (lat_scale && !aligned4(lat_scale)))
    return DSA_ERR_INVALID_ARG;
  const size_t need = ws_bytes_for(want_causal ? DSA_OP_SPARSE_MLA_PREFILL : DSA_OP_SPARSE_MLA_DECODE,
                                   *dims, *cache);
  DSA_TRY(check_ws(ws, ws_bytes, need));
  if (dims->n_q == 0) return DSA_OK;
  return run_mla(q, latent_pages, *cache, idx, *dims, out, lse,
                 static_cast<uint8_t *>(ws) + kStatusBytes, ws_bytes - kStatusBytes, status_of(ws),
                 as_stream(stream), 0, latent8_pages, lat_scale);
}

dsa_status_t indexer_entry(const uint16_t *q_idx, const float *w, const uint16_t *k_idx_pages,
                           const uint8_t *k8_pages, const float *k_scale, const dsa_cache_t *cache,
                           const dsa_dims_t *dims, float *scores, int64_t ld, void *ws,
                           size_t ws_bytes, dsa_stream_t stream);
dsa_status_t forward_entry(const uint16_t *q_idx, const float *w, const uint16_t *k_idx_pages,
                           const uint8_t *k8_pages, const float *k_scale, const uint16_t *q,
                           const uint16_t *latent_pages, const dsa_cache_t *cache,
                           const dsa_dims_t *dims, int32_t *idx_out, float *out, float *lse,
                           void *ws, size_t ws_bytes, dsa_stream_t stream,
                           const uint8_t *latent8_pages = nullptr, const float *lat_scale = nullptr,
                           const void *q_src = nullptr, size_t q_copy_bytes = 0);

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" {

int dsa_version(void) { return 100; }

const char *dsa_last_cuda_error(void) { return g_last_error; }

const char *dsa_status_string(dsa_status_t s) {
  switch (s) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported shape or configuration";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case DSA_ERR_TIMEOUT: return "a bounded device-side wait timed out";
    case DSA_ERR_DEVICE_CHECK: return "a device-side range check failed";
  }
  return "unknown status";
}

size_t dsa_workspace_bytes(dsa_op_t op, const dsa_dims_t *dims, const dsa_cache_t *cache) {
  if (check_dims_common(dims) != DSA_OK) return 0;
  if (op == DSA_OP_INDEXER_SCORES || op == DSA_OP_TOPK || op == DSA_OP_CACHE_APPEND)
    return kStatusBytes;
  if (op == DSA_OP_INDEXER_SCORES_K8) return ws_bytes_for(op, *dims, dsa_cache_t{});
  if (check_mla_dims(*dims) != DSA_OK) return 0;
  if ((op == DSA_OP_ATTENTION_FORWARD || op == DSA_OP_ATTENTION_FORWARD_K8 ||
       op == DSA_OP_ATTENTION_FORWARD_FP8 || op == DSA_OP_ATTENTION_FORWARD_HOST) &&
      (cache == nullptr || check_cache(cache, *dims) != DSA_OK))
    return 0;
  dsa_cache_t empty = {};
  return ws_bytes_for(op, *dims, cache ? *cache : empty);
}

int32_t dsa_forward_launches(dsa_op_t op, const dsa_dims_t *dims, const dsa_cache_t *cache) {
  if (op != DSA_OP_ATTENTION_FORWARD && op != DSA_OP_ATTENTION_FORWARD_K8 &&
      op != DSA_OP_ATTENTION_FORWARD_FP8)
    return -1;
  if (check_dims_common(dims) != DSA_OK || check_indexer_dims(*dims) != DSA_OK ||
      check_mla_dims(*dims) != DSA_OK || check_cache(cache, *dims) != DSA_OK)
    return -1;
  if (dims->n_q == 0) return 0;
  // indexer (+ the E4M3 query split for FP8 keys), top-k, sparse MLA (+ merge)
  return (op == DSA_OP_ATTENTION_FORWARD ? 2 : 3) +
         mla_launch_count(dims->n_q, dims->topk, dims->R, dims->P,
                          op == DSA_OP_ATTENTION_FORWARD_FP8);
}

dsa_status_t dsa_workspace_init(void *ws, size_t ws_bytes, dsa_stream_t stream) {
  DSA_TRY(check_ws(ws, ws_bytes, kStatusBytes));
  if (cudaMemsetAsync(ws, 0, kStatusBytes, as_stream(stream)) != cudaSuccess) return DSA_ERR_CUDA;
  return DSA_OK;
}

dsa_status_t dsa_workspace_check(const void *ws, dsa_stream_t stream, uint32_t *info) {
  if (ws == nullptr) return DSA_ERR_WORKSPACE;
  DevStatus host;
  cudaStream_t s = as_stream(stream);
  if (cudaMemcpyAsync(&host, ws, sizeof(host), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return DSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DSA_ERR_CUDA;
  if (info) *info = host.first;
  if (host.flags & kErrTimeout) return DSA_ERR_TIMEOUT;
  if (host.flags != 0u) return DSA_ERR_DEVICE_CHECK;
  return DSA_OK;
}

dsa_status_t dsa_indexer_scores(const uint16_t *q_idx, const float *w, const uint16_t *k_idx_pages,
                                const dsa_cache_t *cache, const dsa_dims_t *dims, float *scores,
                                int64_t ld, void *ws, size_t ws_bytes, dsa_stream_t stream) {
  return indexer_entry(q_idx, w, k_idx_pages, nullptr, nullptr, cache, dims, scores, ld, ws,
                       ws_bytes, stream);
}

dsa_status_t dsa_indexer_scores_k8(const uint16_t *q_idx, const float *w, const uint8_t *k8_pages,
                                   const float *k_scale, const dsa_cache_t *cache,
                                   const dsa_dims_t *dims, float *scores, int64_t ld, void *ws,
                                   size_t ws_bytes, dsa_stream_t stream) {
  if (k8_pages == nullptr || k_scale == nullptr) return DSA_ERR_INVALID_ARG;
  return indexer_entry(q_idx, w, nullptr, k8_pages, k_scale, cache, dims, scores, ld, ws,
                       ws_bytes, stream);
}

dsa_status_t dsa_topk(const float *scores, int64_t ld, int32_t n_q, const int32_t *valid_len,
                      int32_t causal_base, int32_t k, int32_t *idx, void *ws, size_t ws_bytes,
                      dsa_stream_t stream) {
  if (scores == nullptr || idx == nullptr) return DSA_ERR_INVALID_ARG;
  if (n_q < 0 || k < 1 || ld < 1 || ld > INT32_MAX) return DSA_ERR_INVALID_ARG;
  if (!aligned4(scores) || !aligned4(idx) || (valid_len && !aligned4(valid_len)))
    return DSA_ERR_INVALID_ARG;
  if (valid_len == nullptr && causal_base < -1) return DSA_ERR_INVALID_ARG;
  if (n_q > 262144) return DSA_ERR_UNSUPPORTED;  // grid.x with 8-CTA clusters
  DSA_TRY(check_ws(ws, ws_bytes, kStatusBytes));
  if (n_q == 0) return DSA_OK;
  // without a host-side bound on the lengths, size the kernel for the full row
  const int max_len = static_cast<int>(
      valid_len ? ld : std::min<int64_t>(ld, static_cast<int64_t>(causal_base) + n_q));
  return run_topk(scores, ld, n_q, valid_len, causal_base, k, idx, max_len, status_of(ws),
                  as_stream(stream));
}

dsa_status_t dsa_sparse_mla_decode(const uint16_t *q, const uint16_t *latent_pages,
                                   const dsa_cache_t *cache, const int32_t *idx,
                                   const dsa_dims_t *dims, float *out, float *lse, void *ws,
                                   size_t ws_bytes, dsa_stream_t stream) {
  return mla_entry(q, latent_pages, nullptr, nullptr, cache, idx, dims, out, lse, ws, ws_bytes,
                   stream, 0);
}

dsa_status_t dsa_sparse_mla_prefill(const uint16_t *q, const uint16_t *latent_pages,
                                    const dsa_cache_t *cache, const int32_t *idx,
                                    const dsa_dims_t *dims, float *out, float *lse, void *ws,
                                    size_t ws_bytes, dsa_stream_t stream) {
  return mla_entry(q, latent_pages, nullptr, nullptr, cache, idx, dims, out, lse, ws, ws_bytes,
                   stream, 1);
}

dsa_status_t dsa_sparse_mla_decode_l8(const uint16_t *q, const uint8_t *latent8_pages,
                                      const float *latent_scale, const dsa_cache_t *cache,
                                      const int32_t *idx, const dsa_dims_t *dims, float *out,
                                      float *lse, void *ws, size_t ws_bytes, dsa_stream_t stream) {
  if (latent8_pages == nullptr || latent_scale == nullptr) return DSA_ERR_INVALID_ARG;
  return mla_entry(q, nullptr, latent8_pages, latent_scale, cache, idx, dims, out, lse, ws,
                   ws_bytes, stream, 0);
}

dsa_status_t dsa_sparse_mla_prefill_l8(const uint16_t *q, const uint8_t *latent8_pages,
                                       const float *latent_scale, const dsa_cache_t *cache,
                                       const int32_t *idx, const dsa_dims_t *dims, float *out,
                                       float *lse, void *ws, size_t ws_bytes, dsa_stream_t stream) {
  if (latent8_pages == nullptr || latent_scale == nullptr) return DSA_ERR_INVALID_ARG;
  return mla_entry(q, nullptr, latent8_pages, latent_scale, cache, idx, dims, out, lse, ws,
                   ws_bytes, stream, 1);
}

dsa_status_t dsa_attention_forward(const uint16_t *q_idx, const float *w,
                                   const uint16_t *k_idx_pages, const uint16_t *q,
                                   const uint16_t *latent_pages, const dsa_cache_t *cache,
                                   const dsa_dims_t *dims, int32_t *idx_out, float *out,
                                   float *lse, void *ws, size_t ws_bytes, dsa_stream_t stream) {
  return forward_entry(q_idx, w, k_idx_pages, nullptr, nullptr, q, latent_pages, cache, dims,
                       idx_out, out, lse, ws, ws_bytes, stream);
}

dsa_status_t dsa_attention_forward_host(const uint16_t *q_idx_h, const float *w_h,
                                        const uint16_t *k_idx_pages, const uint16_t *q_h,
                                        const uint16_t *latent_pages, const dsa_cache_t *cache_h,
                                        const dsa_dims_t *dims, int32_t *idx_h, float *out_h,
                                        float *lse_h, void *ws, size_t ws_bytes,
                                        dsa_stream_t stream) {
  DSA_TRY(check_dims_common(dims));
  DSA_TRY(check_indexer_dims(*dims));
  DSA_TRY(check_mla_dims(*dims));
  DSA_TRY(check_cache(cache_h, *dims));
  if (q_idx_h == nullptr || w_h == nullptr || k_idx_pages == nullptr || q_h == nullptr ||
      latent_pages == nullptr || out_h == nullptr || lse_h == nullptr)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(k_idx_pages) || !aligned16(latent_pages)) return DSA_ERR_INVALID_ARG;
  const dsa_dims_t &d = *dims;
  const dsa_cache_t &ch = *cache_h;
  const size_t fwd = ws_bytes_for(DSA_OP_ATTENTION_FORWARD, d, ch);  // a multiple of 256
  DSA_TRY(check_ws(ws, ws_bytes, fwd + host_stage_bytes(d, ch)));
  if (d.n_q == 0) return DSA_OK;
  const HostStage h = host_stage_sizes(d, ch);
  uint8_t *p = static_cast<uint8_t *>(ws) + fwd;
  auto take = [&p](size_t bytes) {
    uint8_t *r = p;
    p += align256(bytes);
    return r;
  };
  uint16_t *q_idx = reinterpret_cast<uint16_t *>(take(h.q_idx));
  float *w = reinterpret_cast<float *>(take(h.w));
  uint16_t *q = reinterpret_cast<uint16_t *>(take(h.q));
  int32_t *seq_lens = reinterpret_cast<int32_t *>(take(h.seq_lens));
  int32_t *block_table = reinterpret_cast<int32_t *>(take(h.block_table));
  int32_t *idx = reinterpret_cast<int32_t *>(take(h.idx));
  float *out = reinterpret_cast<float *>(take(h.out));
  float *lse = reinterpret_cast<float *>(take(h.lse));
  cudaStream_t s = as_stream(stream);
  // Host buffers the device can address (pinned and mapped) move with one
  // kernel each way; any other buffer with its own cudaMemcpyAsync.
  CopyList in{}, out_l{};
  bool ok = true;
  auto add = [&](CopyList &l, const void *src, void *dst, size_t bytes, const void *host,
                 bool to_device) {
    void *mapped = mapped_host(host);
    if (mapped != nullptr) {
      CopyPiece &pc = l.piece[l.n++];
      pc.src = to_device ? mapped : src;
      pc.dst = to_device ? dst : mapped;
      pc.bytes = bytes;
    } else if (cudaMemcpyAsync(dst, src, bytes,
                               to_device ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToHost,
                               s) != cudaSuccess) {
      ok = false;
    }
  };
  add(in, q_idx_h, q_idx, h.q_idx, q_idx_h, true);
  add(in, w_h, w, h.w, w_h, true);
  // The attention query (most of the input bytes) is read only by the MLA:
  // from mapped host memory the indexer's copy warps move it while the keys
  // are scanned, and the host link is otherwise idle
  const void *q_mapped = mapped_host(q_h);
  const bool q_by_indexer = q_mapped != nullptr && h.q % 16 == 0 &&
                            (reinterpret_cast<uintptr_t>(q_mapped) & 15u) == 0;
  if (!q_by_indexer) add(in, q_h, q, h.q, q_h, true);
  add(in, ch.seq_lens, seq_lens, h.seq_lens, ch.seq_lens, true);
  add(in, ch.block_table, block_table, h.block_table, ch.block_table, true);
  if (!ok) return DSA_ERR_CUDA;
  DSA_TRY(launch_copy_pieces(in, s));
  dsa_cache_t cd = ch;
  cd.seq_lens = seq_lens;
  cd.block_table = block_table;
  DSA_TRY(forward_entry(q_idx, w, k_idx_pages, nullptr, nullptr, q, latent_pages, &cd, dims,
                        idx_h ? idx : nullptr, out, lse, ws, fwd, stream, nullptr, nullptr,
                        q_by_indexer ? q_mapped : nullptr, h.q));
  if (idx_h) add(out_l, idx, idx_h, h.idx, idx_h, false);
  add(out_l, out, out_h, h.out, out_h, false);
  add(out_l, lse, lse_h, h.lse, lse_h, false);
  if (!ok) return DSA_ERR_CUDA;
  return launch_copy_pieces(out_l, s);
}

dsa_status_t dsa_attention_forward_k8(const uint16_t *q_idx, const float *w,
                                      const uint8_t *k8_pages, const float *k_scale,
                                      const uint16_t *q, const uint16_t *latent_pages,
                                      const dsa_cache_t *cache, const dsa_dims_t *dims,
                                      int32_t *idx_out, float *out, float *lse, void *ws,
                                      size_t ws_bytes, dsa_stream_t stream) {
  if (k8_pages == nullptr || k_scale == nullptr) return DSA_ERR_INVALID_ARG;
  return forward_entry(q_idx, w, nullptr, k8_pages, k_scale, q, latent_pages, cache, dims,
                       idx_out, out, lse, ws, ws_bytes, stream);
}

dsa_status_t dsa_attention_forward_fp8(const uint16_t *q_idx, const float *w,
                                       const uint8_t *k8_pages, const float *k_scale,
                                       const uint16_t *q, const uint8_t *latent8_pages,
                                       const float *latent_scale, const dsa_cache_t *cache,
                                       const dsa_dims_t *dims, int32_t *idx_out, float *out,
                                       float *lse, void *ws, size_t ws_bytes, dsa_stream_t stream) {
  if (k8_pages == nullptr || k_scale == nullptr || latent8_pages == nullptr ||
      latent_scale == nullptr)
    return DSA_ERR_INVALID_ARG;
  return forward_entry(q_idx, w, nullptr, k8_pages, k_scale, q, nullptr, cache, dims, idx_out,
                       out, lse, ws, ws_bytes, stream, latent8_pages, latent_scale);
}

size_t dsa_cp_workspace_bytes(int32_t ranks, int32_t n_q, int32_t k) {
  if (ranks < 1 || n_q < 0 || k < 1) return 0;
  const int64_t ld = (static_cast<int64_t>(ranks) * k + 3) & ~static_cast<int64_t>(3);
  return kStatusBytes + align256(static_cast<size_t>(n_q) * ld * 4) +
         align256(static_cast<size_t>(n_q) * k * 4) + align256(static_cast<size_t>(n_q) * 4);
}

dsa_status_t dsa_cp_candidates(const float *scores, int64_t ld, int32_t n_q, const int32_t *idx_local,
                               int32_t k, const int32_t *offsets, float *cand_scores,
                               int32_t *cand_idx, void *ws, size_t ws_bytes, dsa_stream_t stream) {
  if (n_q < 0 || k < 1 || ld < 1) return DSA_ERR_INVALID_ARG;
  if (scores == nullptr || idx_local == nullptr || offsets == nullptr || cand_scores == nullptr ||
      cand_idx == nullptr)
    return DSA_ERR_INVALID_ARG;
  if (!aligned4(scores) || !aligned4(idx_local) || !aligned4(offsets) || !aligned4(cand_scores) ||
      !aligned4(cand_idx))
    return DSA_ERR_INVALID_ARG;
  DSA_TRY(check_ws(ws, ws_bytes, kStatusBytes));
  if (n_q == 0) return DSA_OK;
  return launch_cp_candidates(scores, ld, n_q, idx_local, k, offsets, cand_scores, cand_idx,
                              as_stream(stream));
}

dsa_status_t dsa_cp_select(const float *all_scores, const int32_t *all_idx, int32_t ranks,
                           int32_t n_q, int32_t k, const int32_t *my_offsets,
                           const int32_t *my_lens, int32_t *gidx, int32_t *own_idx, void *ws,
                           size_t ws_bytes, dsa_stream_t stream) {
  if (ranks < 1 || n_q < 0 || k < 1 || k > 65536) return DSA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(ranks) * k > (1 << 24)) return DSA_ERR_UNSUPPORTED;
  if (all_scores == nullptr || all_idx == nullptr || my_offsets == nullptr || my_lens == nullptr ||
      gidx == nullptr || own_idx == nullptr)
    return DSA_ERR_INVALID_ARG;
  if (!aligned4(all_scores) || !aligned4(all_idx) || !aligned4(my_offsets) || !aligned4(my_lens) ||
      !aligned4(gidx) || !aligned4(own_idx))
    return DSA_ERR_INVALID_ARG;
  DSA_TRY(check_ws(ws, ws_bytes, dsa_cp_workspace_bytes(ranks, n_q, k)));
  if (n_q == 0) return DSA_OK;
  const int64_t ld = (static_cast<int64_t>(ranks) * k + 3) & ~static_cast<int64_t>(3);
  uint8_t *base = static_cast<uint8_t *>(ws) + kStatusBytes;
  float *packed = reinterpret_cast<float *>(base);
  int32_t *pos = reinterpret_cast<int32_t *>(base + align256(static_cast<size_t>(n_q) * ld * 4));
  int32_t *vlen = reinterpret_cast<int32_t *>(reinterpret_cast<uint8_t *>(pos) +
                                              align256(static_cast<size_t>(n_q) * k * 4));
  cudaStream_t s = as_stream(stream);
  DSA_TRY(launch_cp_pack(all_scores, ranks, n_q, k, ld, packed, vlen, s));
  DSA_TRY(run_topk(packed, ld, n_q, vlen, 0, k, pos, static_cast<int>(ranks * k), status_of(ws), s));
  return launch_cp_select(pos, all_idx, ranks, n_q, k, my_offsets, my_lens, gidx, own_idx, s);
}

dsa_status_t dsa_cp_merge(const float *outs, const float *lses, int32_t ranks, int32_t n_q,
                          int32_t H, int32_t dv, float *out, float *lse, void *ws, size_t ws_bytes,
                          dsa_stream_t stream) {
  if (ranks < 1 || n_q < 0 || H < 1 || H > 65535 || dv < 1) return DSA_ERR_INVALID_ARG;
  if (ranks > 1024) return DSA_ERR_UNSUPPORTED;
  if (outs == nullptr || lses == nullptr || out == nullptr || lse == nullptr)
    return DSA_ERR_INVALID_ARG;
  if (!aligned4(outs) || !aligned4(lses) || !aligned4(out) || !aligned4(lse))
    return DSA_ERR_INVALID_ARG;
  DSA_TRY(check_ws(ws, ws_bytes, kStatusBytes));
  if (n_q == 0) return DSA_OK;
  return launch_cp_merge(outs, lses, ranks, n_q, H, dv, out, lse, as_stream(stream));
}

}  // extern "C"

namespace dsa {
namespace {

// the indexer entry for bf16 keys (k_idx_pages) or E4M3 keys (k8_pages + k_scale)
dsa_status_t indexer_entry(const uint16_t *q_idx, const float *w, const uint16_t *k_idx_pages,
                           const uint8_t *k8_pages, const float *k_scale, const dsa_cache_t *cache,
                           const dsa_dims_t *dims, float *scores, int64_t ld, void *ws,
                           size_t ws_bytes, dsa_stream_t stream) {
  DSA_TRY(check_dims_common(dims));
  DSA_TRY(check_indexer_dims(*dims));
  DSA_TRY(check_cache(cache, *dims));
  const void *keys = k8_pages ? static_cast<const void *>(k8_pages) : k_idx_pages;
  if (q_idx == nullptr || w == nullptr || keys == nullptr || scores == nullptr)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(keys) || !aligned16(scores) || !aligned4(w) ||
      (k_scale && !aligned16(k_scale)))
    return DSA_ERR_INVALID_ARG;
  if (k8_pages && dims->D_I != 128) return DSA_ERR_UNSUPPORTED;
  if (ld < max_keys(*dims, *cache) || ld % 4 != 0 || ld <= 0) return DSA_ERR_INVALID_ARG;
  DSA_TRY(check_ws(ws, ws_bytes,
                   k8_pages ? ws_bytes_for(DSA_OP_INDEXER_SCORES_K8, *dims, *cache) : kStatusBytes));
  if (dims->n_q == 0) return DSA_OK;
  return run_indexer(q_idx, w, k_idx_pages, *cache, *dims, scores, ld, status_of(ws),
                     as_stream(stream), k8_pages, k_scale, static_cast<uint8_t *>(ws) + kStatusBytes);
}

// the whole step for bf16 keys (k_idx_pages) or E4M3 keys (k8_pages + k_scale)
dsa_status_t forward_entry(const uint16_t *q_idx, const float *w, const uint16_t *k_idx_pages,
                           const uint8_t *k8_pages, const float *k_scale, const uint16_t *q,
                           const uint16_t *latent_pages, const dsa_cache_t *cache,
                           const dsa_dims_t *dims, int32_t *idx_out, float *out, float *lse,
                           void *ws, size_t ws_bytes, dsa_stream_t stream,
                           const uint8_t *latent8_pages, const float *lat_scale,
                           const void *q_src, size_t q_copy_bytes) {
  DSA_TRY(check_dims_common(dims));
  DSA_TRY(check_indexer_dims(*dims));
  DSA_TRY(check_mla_dims(*dims));
  DSA_TRY(check_cache(cache, *dims));
  const void *keys = k8_pages ? static_cast<const void *>(k8_pages) : k_idx_pages;
  const void *lat = latent8_pages ? static_cast<const void *>(latent8_pages) : latent_pages;
  if (q_idx == nullptr || w == nullptr || keys == nullptr || q == nullptr || lat == nullptr ||
      out == nullptr || lse == nullptr)
    return DSA_ERR_INVALID_ARG;
  if ((lat_scale && !aligned4(lat_scale))) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(keys) || !aligned16(q) || !aligned16(lat) ||
      !aligned4(w) || !aligned4(out) || !aligned4(lse) || (idx_out && !aligned4(idx_out)) ||
      (k_scale && !aligned16(k_scale)))
    return DSA_ERR_INVALID_ARG;
  if (k8_pages && dims->D_I != 128) return DSA_ERR_UNSUPPORTED;
  const dsa_dims_t &d = *dims;
  const dsa_cache_t &c = *cache;
  DSA_TRY(check_ws(ws, ws_bytes,
                   ws_bytes_for(k8_pages ? DSA_OP_ATTENTION_FORWARD_K8 : DSA_OP_ATTENTION_FORWARD,
                                d, c)));
  if (d.n_q == 0) return DSA_OK;

  // FP8 keys: the query terms right after the status block, the rest shifted
  uint8_t *k8_region = static_cast<uint8_t *>(ws) + kStatusBytes;
  uint8_t *base = static_cast<uint8_t *>(ws) + (k8_pages ? k8_region_bytes(d) : 0);
  DevStatus *st = status_of(ws);
  const int64_t ld = scores_ld(d, c);
  float *scores = reinterpret_cast<float *>(base + kStatusBytes);
  int32_t *idx_ws = reinterpret_cast<int32_t *>(
      base + kStatusBytes + align256(static_cast<size_t>(d.n_q) * ld * 4));
  uint8_t *scratch = reinterpret_cast<uint8_t *>(idx_ws) + align256(static_cast<size_t>(d.n_q) * d.topk * 4);
  const size_t scratch_bytes = ws_bytes - static_cast<size_t>(scratch - static_cast<uint8_t *>(ws));
  int32_t *idx = idx_out ? idx_out : idx_ws;
  cudaStream_t s = as_stream(stream);

  // q_src: the attention query is still to be copied into q (q_copy_bytes),
  // which the indexer does under its key scan (bf16 keys only)
  DSA_TRY(run_indexer(q_idx, w, k_idx_pages, c, d, scores, ld, st, s, k8_pages, k_scale,
                      k8_region, q_src, const_cast<uint16_t *>(q), q_src ? q_copy_bytes : 0));
  DSA_TRY(run_topk(scores, ld, d.n_q, d.causal ? nullptr : c.seq_lens, d.q_pos0, d.topk, idx,
                   static_cast<int>(max_keys(d, c)), st, s));
  return run_mla(q, latent_pages, c, idx, d, out, lse, scratch, scratch_bytes, st, s,
                 /*early_q=*/1, latent8_pages, lat_scale);
}

}  // namespace
}  // namespace dsa

extern "C" {

dsa_status_t dsa_cache_append(const uint16_t *k_idx_new, const uint16_t *latent_new,
                              uint16_t *k_idx_pages, uint16_t *latent_pages,
                              const dsa_cache_t *cache, const dsa_dims_t *dims, void *ws,
                              size_t ws_bytes, dsa_stream_t stream) {
  DSA_TRY(check_dims_common(dims));
  const dsa_dims_t &d = *dims;
  if (d.D_I != 32 && d.D_I != 64 && d.D_I != 128) return DSA_ERR_UNSUPPORTED;
  if (d.R < 64 || d.R > 512 || d.R % 64 != 0) return DSA_ERR_UNSUPPORTED;
  if (d.P < 0 || d.P % 16 != 0 || d.R + d.P > 576) return DSA_ERR_UNSUPPORTED;
  DSA_TRY(check_cache(cache, d));
  if (k_idx_new == nullptr || latent_new == nullptr || k_idx_pages == nullptr ||
      latent_pages == nullptr)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(k_idx_new) || !aligned16(latent_new) || !aligned16(k_idx_pages) ||
      !aligned16(latent_pages))
    return DSA_ERR_INVALID_ARG;
  DSA_TRY(check_ws(ws, ws_bytes, kStatusBytes));
  if (d.n_q == 0) return DSA_OK;
  AppendLaunch a;
  a.k_new = k_idx_new;
  a.lat_new = latent_new;
  a.k_pages = k_idx_pages;
  a.lat_pages = latent_pages;
  a.seq_lens = cache->seq_lens;
  a.block_table = cache->block_table;
  a.n_q = d.n_q;
  a.D_I = d.D_I;
  a.W = d.R + d.P;
  a.causal = d.causal;
  a.q_pos0 = d.q_pos0;
  a.max_pages = cache->max_pages;
  a.num_pages = cache->num_pages;
  a.status = status_of(ws);
  return launch_append(a, as_stream(stream));
}

dsa_status_t dsa_absorb_query(const uint16_t *q_nope, const uint16_t *q_rope, const uint16_t *w_uk,
                              uint16_t *q_abs, int32_t n_q, int32_t H, int32_t d_nope, int32_t R,
                              int32_t P, void *ws, size_t ws_bytes, dsa_stream_t stream) {
  if (n_q < 0 || H < 1 || H > 128) return DSA_ERR_INVALID_ARG;
  if (d_nope < 64 || d_nope > 512 || d_nope % 64 != 0) return DSA_ERR_UNSUPPORTED;
  if (R < 64 || R > 512 || R % 64 != 0) return DSA_ERR_UNSUPPORTED;
  if (P < 0 || P % 16 != 0 || R + P > 576) return DSA_ERR_UNSUPPORTED;
  if (q_nope == nullptr || w_uk == nullptr || q_abs == nullptr || (P > 0 && q_rope == nullptr))
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_nope) || !aligned16(w_uk) || !aligned16(q_abs) ||
      (P > 0 && !aligned16(q_rope)))
    return DSA_ERR_INVALID_ARG;
  DSA_TRY(check_ws(ws, ws_bytes, kStatusBytes));
  if (n_q == 0) return DSA_OK;
  AbsorbLaunch a = {};
  a.project = false;
  a.x = q_nope;
  a.rope = q_rope;
  a.w = w_uk;
  a.out_bf16 = q_abs;
  a.n = n_q;
  a.H = H;
  a.K = d_nope;
  a.M = R;
  a.P = P;
  a.status = status_of(ws);
  return launch_absorb(a, as_stream(stream));
}

dsa_status_t dsa_project_values(const float *o_lat, const uint16_t *w_uv, float *v_out,
                                int32_t n_q, int32_t H, int32_t R, int32_t d_v, void *ws,
                                size_t ws_bytes, dsa_stream_t stream) {
  if (n_q < 0 || H < 1 || H > 128) return DSA_ERR_INVALID_ARG;
  if (R < 64 || R > 512 || R % 64 != 0) return DSA_ERR_UNSUPPORTED;
  if (d_v < 64 || d_v > 512 || d_v % 64 != 0) return DSA_ERR_UNSUPPORTED;
  if (o_lat == nullptr || w_uv == nullptr || v_out == nullptr) return DSA_ERR_INVALID_ARG;
  if (!aligned16(o_lat) || !aligned16(w_uv) || !aligned4(v_out)) return DSA_ERR_INVALID_ARG;
  DSA_TRY(check_ws(ws, ws_bytes, kStatusBytes));
  if (n_q == 0) return DSA_OK;
  AbsorbLaunch a = {};
  a.project = true;
  a.xf = o_lat;
  a.w = w_uv;
  a.out_f32 = v_out;
  a.n = n_q;
  a.H = H;
  a.K = R;
  a.M = d_v;
  a.P = 0;
  a.status = status_of(ws);
  return launch_absorb(a, as_stream(stream));
}

}  // extern "C"
