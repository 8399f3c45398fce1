// dsa_api.cu -- the C ABI (include/dsa.h): argument validation, workspace
// sizing, the IndexCache layer loop and error reporting.  All compute runs in
// the kernels of indexer_topk.cu and sparse_attn.cu.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "dsa_internal.h"
#include "dsa_ptx.cuh"

namespace dsa {

__device__ unsigned int g_dsa_error = 0;

namespace {
std::string g_last_error = "no error";
std::atomic<long long> g_indexer_launches{0};

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}
}  // namespace

dsa_status set_error(dsa_status st, const std::string& msg) {
  g_last_error = msg;
  return st;
}

bool encode_tiled_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                     uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0, uint32_t box1,
                     CUtensorMapSwizzle swizzle, CUtensorMapDataType dtype) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  const cuuint32_t box[3] = {box0, box1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, dtype, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tiled_2d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1,
                     uint64_t stride1_bytes, uint32_t box0, uint32_t box1,
                     CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {d0, d1};
  const cuuint64_t strides[1] = {stride1_bytes};
  const cuuint32_t box[2] = {box0, box1};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

unsigned int* device_error_word() {
  static unsigned int* cache[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dsa_error) != cudaSuccess) return nullptr;
    cache[dev] = static_cast<unsigned int*>(p);
  }
  return cache[dev];
}

cudaError_t ensure_smem_limit(const void* func, int bytes) {
  static std::mutex mu;
  static std::vector<std::pair<std::pair<int, const void*>, int>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (auto& d : done)
    if (d.first.first == dev && d.first.second == func && d.second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.push_back({{dev, func}, bytes});
  return e;
}

int device_sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    cache[dev] = n;
  }
  return cache[dev];
}

// Self-test of the bounded-wait path: one CTA waits on an mbarrier that
// nothing ever arrives on, gives up after `limit` cycles, and records the
// expiry in the device error word the way every kernel's waits do.
__global__ void selftest_wait_kernel(unsigned int* err, long long limit) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  const uint32_t a = smem_u32(&bar);
  const long long t0 = clock64();
  bool done = false;
  while (!(done = mbar_try_wait(a, 0)) && clock64() - t0 < limit) {
  }
  if (!done && threadIdx.x == 0) atomicOr(err, 1u);
}

// Checks that index rows have the canonical form dsa_indexer_topk writes
// ([IDX] §1, §4: S_t is a subset of {s : 0 <= s < t} of size min(t, k)):
// the first min(t, k) entries strictly ascending in [0, t), then -1.  One warp per row; each bad row adds 1 to *bad_rows.
__global__ void check_indices_kernel(const int32_t* __restrict__ idx, int Lq, int start_pos, int k,
                                     int* bad_rows) {
  const size_t row = blockIdx.x;
  const int t = start_pos + static_cast<int>(row % Lq);
  const int n = min(t, k);
  const int32_t* r = idx + row * k;
  bool bad = false;
  for (int e = threadIdx.x; e < k; e += 32) {
    const int32_t v = r[e];
    if (e < n) {
      bad |= v < 0 || v >= t;
      if (e > 0) bad |= v <= r[e - 1];
    } else {
      bad |= v != -1;
    }
  }
  if (__any_sync(0xffffffffu, bad) && threadIdx.x == 0) atomicAdd(bad_rows, 1);
}

// Index rows when every row sees at most k positions (t <= k): TopK keeps
// all of P_t = {s : 0 <= s < t} ([IDX] §1, §4), so row t is 0, 1, ..., t-1
// and then -1, and no score needs computing.  This is the short-prefill case
// in which a sparse layer reads exactly what masked dense attention reads.
__global__ void full_visible_rows_kernel(int32_t* __restrict__ idx, int64_t n, int Lq, int start_pos, int k) {
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = e / k;
    const int r = static_cast<int>(e % k);
    const int t = start_pos + static_cast<int>(row % Lq);
    idx[e] = r < t ? r : -1;
  }
}

// Contract of a variable-length batch (include/dsa.h), one thread per
// sequence: offsets start at 0, never decrease, end at the totals; lengths
// within the bounds; every query row within its cache (t <= Lk_b).
__global__ void check_varlen_kernel(const int* __restrict__ cu_q, const int* __restrict__ cu_k,
                                    const int* __restrict__ sp, int B, int total_q, int total_k, int max_Lq,
                                    int max_Lk, int* bad) {
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < B; b += gridDim.x * blockDim.x) {
    const int q0 = cu_q[b], q1 = cu_q[b + 1], k0 = cu_k[b], k1 = cu_k[b + 1];
    bool ok = q1 >= q0 && k1 >= k0 && q1 - q0 <= max_Lq && k1 - k0 <= max_Lk && sp[b] >= 0 &&
              static_cast<long long>(sp[b]) + (q1 - q0) - 1 <= static_cast<long long>(k1 - k0);
    if (b == 0) ok = ok && q0 == 0 && k0 == 0;
    if (b == B - 1) ok = ok && q1 == total_q && k1 == total_k;
    if (!ok) atomicAdd(bad, 1);
  }
}

}  // namespace dsa

using namespace dsa;

namespace {

dsa_status check_indexer_args(const dsa_bf16* q_idx, const dsa_bf16* k_idx, const float* w,
                              int B, int Lq, int Lk, int start_pos, int H, int d, int k,
                              const int32_t* idx) {
  if (!q_idx || !k_idx || !w || !idx)
    return set_error(DSA_ERR_INVALID_ARG, "dsa_indexer_topk: null pointer");
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w) || !aligned16(idx))
    return set_error(DSA_ERR_INVALID_ARG, "dsa_indexer_topk: pointers must be 16-byte aligned");
  if (B < 1 || Lq < 1 || Lk < 1 || start_pos < 0 || k < 1)
    return set_error(DSA_ERR_INVALID_ARG, "dsa_indexer_topk: sizes must be positive");
  if (static_cast<long long>(start_pos) + Lq - 1 > Lk)
    return set_error(DSA_ERR_INVALID_ARG, "dsa_indexer_topk: start_pos + Lq - 1 exceeds Lk");
  if (!indexer_supported(H, d, k))
    return set_error(DSA_ERR_UNSUPPORTED,
                     "dsa_indexer_topk: need H_I in {4,8,16,32,64}, d_I in {32,64,128}, k <= 2048");
  if (static_cast<long long>(Lq) * H > (1ll << 31) - 1 || static_cast<long long>(B) * Lq * k > (1ll << 40))
    return set_error(DSA_ERR_UNSUPPORTED, "dsa_indexer_topk: tensor too large");
  return DSA_OK;
}

dsa_status check_varlen_host(const dsa_varlen* vl, VarlenArgs* out) {
  if (!vl) return set_error(DSA_ERR_INVALID_ARG, "varlen: null batch descriptor");
  if (!vl->cu_q || !vl->cu_k || !vl->start_pos)
    return set_error(DSA_ERR_INVALID_ARG, "varlen: null offset or position array");
  if ((reinterpret_cast<uintptr_t>(vl->cu_q) | reinterpret_cast<uintptr_t>(vl->cu_k) |
       reinterpret_cast<uintptr_t>(vl->start_pos)) & 3u)
    return set_error(DSA_ERR_INVALID_ARG, "varlen: offset arrays must be 4-byte aligned");
  if (vl->B < 1 || vl->total_q < 1 || vl->total_k < 1 || vl->max_Lq < 1 || vl->max_Lk < 1)
    return set_error(DSA_ERR_INVALID_ARG, "varlen: sizes must be positive");
  if (vl->max_Lq > vl->total_q || vl->max_Lk > vl->total_k)
    return set_error(DSA_ERR_INVALID_ARG, "varlen: a per-sequence bound exceeds the total");
  if (out) *out = VarlenArgs{vl->cu_q, vl->cu_k, vl->start_pos, vl->total_q, vl->total_k};
  return DSA_OK;
}

}  // namespace

extern "C" {

const char* dsa_last_error(void) { return g_last_error.c_str(); }

long long dsa_indexer_launch_count(void) { return g_indexer_launches.load(); }

size_t dsa_indexer_topk_workspace(int B, int Lq, int Lk, int start_pos, int H_I, int d_I, int k) {
  if (B < 1 || Lq < 1 || k < 1 || start_pos < 0) return 0;
  // decode rows keep one score key per cached position instead
  if (decode_indexer_applies(Lq, Lk, start_pos, H_I, d_I)) return decode_indexer_ws_bytes(B, Lk);
  return indexer_plan(B, Lq, Lk, start_pos, std::min(k, 2048)).total_bytes;
}

dsa_status dsa_indexer_topk(const dsa_bf16* q_idx, const dsa_bf16* k_idx, const float* w, int B,
                            int Lq, int Lk, int start_pos, int H_I, int d_I, int k, int32_t* idx,
                            void* ws, size_t ws_bytes, void* stream) {
  dsa_status st = check_indexer_args(q_idx, k_idx, w, B, Lq, Lk, start_pos, H_I, d_I, k, idx);
  if (st != DSA_OK) return st;
  if (!ws || !aligned16(ws)) return set_error(DSA_ERR_WORKSPACE, "dsa_indexer_topk: null or misaligned workspace");
  if (static_cast<long long>(start_pos) + Lq - 1 <= k) {
    const int64_t n = static_cast<int64_t>(B) * Lq * k;
    const int sms = device_sm_count();
    if (sms <= 0) return set_error(DSA_ERR_CUDA, "cannot query the device SM count");
    const unsigned blocks = static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, 8ll * sms)));
    full_visible_rows_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(idx, n, Lq, start_pos, k);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("index rows launch: ") + cudaGetErrorString(e));
    g_indexer_launches.fetch_add(1);
    return DSA_OK;
  }
  st = indexer_topk_launch(q_idx, k_idx, w, B, Lq, Lk, start_pos, H_I, d_I, k, idx, ws, ws_bytes,
                           static_cast<cudaStream_t>(stream));
  if (st == DSA_OK) g_indexer_launches.fetch_add(1);
  return st;
}

size_t dsa_sparse_attn_workspace(int B, int Lq, int n_h, int D_v, int k) {
  if (B < 1 || Lq < 1 || n_h < 1 || D_v < 1 || k < 1) return 0;
  return sparse_attn_ws_bytes(B, Lq, n_h, D_v, k);
}

dsa_status dsa_sparse_attn(const dsa_bf16* q, const dsa_bf16* kbuf, int64_t k_row_stride,
                           const dsa_bf16* vbuf, int64_t v_row_stride, const int32_t* idx, int B,
                           int Lq, int Lk, int start_pos, int n_h, int D_qk, int D_v, int k,
                           float scale, dsa_bf16* out, float* lse, void* ws, size_t ws_bytes,
                           void* stream) {
  if (!q || !kbuf || !vbuf || !idx || !out)
    return set_error(DSA_ERR_INVALID_ARG, "dsa_sparse_attn: null pointer");
  if (!aligned16(q) || !aligned16(kbuf) || !aligned16(vbuf) || !aligned16(idx) || !aligned16(out) ||
      (lse && !aligned16(lse)))
    return set_error(DSA_ERR_INVALID_ARG, "dsa_sparse_attn: pointers must be 16-byte aligned");
  if (B < 1 || Lq < 1 || Lk < 1 || start_pos < 0 || n_h < 1 || D_qk < 1 || D_v < 1 || k < 1)
    return set_error(DSA_ERR_INVALID_ARG, "dsa_sparse_attn: sizes must be positive");
  if (static_cast<long long>(start_pos) + Lq - 1 > Lk)
    return set_error(DSA_ERR_INVALID_ARG, "dsa_sparse_attn: start_pos + Lq - 1 exceeds Lk");
  if (k_row_stride < D_qk || v_row_stride < D_v || (k_row_stride % 8) || (v_row_stride % 8))
    return set_error(DSA_ERR_INVALID_ARG, "dsa_sparse_attn: row strides must cover the row and be multiples of 8");
  return sparse_attn_launch(q, kbuf, k_row_stride, vbuf, v_row_stride, idx, B, Lq, Lk, start_pos,
                            n_h, D_qk, D_v, k, scale, out, lse, ws, ws_bytes,
                            static_cast<cudaStream_t>(stream));
}

size_t indexcache_forward_workspace(const dsa_dims* d) {
  if (!d) return 0;
  return std::max(dsa_indexer_topk_workspace(d->B, d->Lq, d->Lk, d->start_pos, d->H_I, d->d_I, d->k),
                  dsa_sparse_attn_workspace(d->B, d->Lq, d->n_h, d->D_v, d->k));
}

dsa_status indexcache_forward(const char* pattern, int n_layers, const dsa_layer_io* layers,
                              const dsa_dims* dims, int32_t* idx_cache, void* ws, size_t ws_bytes,
                              void* stream) {
  // [IC] §1.1: layer roles are F (own indexer) or S (reuse); the first layer
  // must be F so that S layers always find an index tensor.
  if (!pattern || n_layers < 1) return set_error(DSA_ERR_BAD_PATTERN, "indexcache_forward: empty pattern");
  if (pattern[0] != 'F')
    return set_error(DSA_ERR_BAD_PATTERN, "indexcache_forward: the first layer must be 'F'");
  for (int l = 0; l < n_layers; ++l)
    if (pattern[l] != 'F' && pattern[l] != 'S')
      return set_error(DSA_ERR_BAD_PATTERN, "indexcache_forward: pattern entries must be 'F' or 'S'");
  if (!layers || !dims || !idx_cache)
    return set_error(DSA_ERR_INVALID_ARG, "indexcache_forward: null pointer");
  const dsa_dims& d = *dims;
  if (ws_bytes < indexcache_forward_workspace(dims))
    return set_error(DSA_ERR_WORKSPACE, "indexcache_forward: workspace too small");
  // Validate every layer before enqueueing anything.
  for (int l = 0; l < n_layers; ++l) {
    const dsa_layer_io& L = layers[l];
    if (pattern[l] == 'F') {
      dsa_status st = check_indexer_args(L.q_idx, L.k_idx, L.w, d.B, d.Lq, d.Lk, d.start_pos,
                                         d.H_I, d.d_I, d.k, idx_cache);
      if (st != DSA_OK) return st;
    }
    if (!L.q || !L.kbuf || !L.vbuf || !L.out)
      return set_error(DSA_ERR_INVALID_ARG, "indexcache_forward: null attention pointer");
  }
  // [IC] §1.2, Figure 2: F layers refresh the cache, every layer attends
  // with its own q/K/V through the cached positions.
  for (int l = 0; l < n_layers; ++l) {
    const dsa_layer_io& L = layers[l];
    if (pattern[l] == 'F') {
      dsa_status st = dsa_indexer_topk(L.q_idx, L.k_idx, L.w, d.B, d.Lq, d.Lk, d.start_pos, d.H_I,
                                       d.d_I, d.k, idx_cache, ws, ws_bytes, stream);
      if (st != DSA_OK) return st;
    }
    dsa_status st = dsa_sparse_attn(L.q, L.kbuf, d.k_row_stride, L.vbuf, d.v_row_stride, idx_cache,
                                    d.B, d.Lq, d.Lk, d.start_pos, d.n_h, d.D_qk, d.D_v, d.k,
                                    d.scale, L.out, L.lse, ws, ws_bytes, stream);
    if (st != DSA_OK) return st;
  }
  return DSA_OK;
}

size_t dsa_indexer_topk_varlen_workspace(const dsa_varlen* vl, int H_I, int d_I, int k) {
  if (check_varlen_host(vl, nullptr) != DSA_OK || k < 1) return 0;
  return indexer_varlen_ws_bytes(vl->B, vl->max_Lq, vl->max_Lk, vl->total_q, H_I, d_I, k);
}

dsa_status dsa_indexer_topk_varlen(const dsa_bf16* q_idx, const dsa_bf16* k_idx, const float* w,
                                   const dsa_varlen* vl, int H_I, int d_I, int k, int32_t* idx, void* ws,
                                   size_t ws_bytes, void* stream) {
  VarlenArgs va{};
  dsa_status st = check_varlen_host(vl, &va);
  if (st != DSA_OK) return st;
  // the per-sequence limits of dsa_indexer_topk, on the batch's bounds
  st = check_indexer_args(q_idx, k_idx, w, 1, vl->max_Lq, vl->max_Lk, 0, H_I, d_I, k, idx);
  if (st != DSA_OK) return st;
  if (static_cast<long long>(vl->total_q) * H_I > (1ll << 31) - 1 ||
      static_cast<long long>(vl->total_q) * k > (1ll << 40))
    return set_error(DSA_ERR_UNSUPPORTED, "dsa_indexer_topk_varlen: tensor too large");
  if (!ws || !aligned16(ws)) return set_error(DSA_ERR_WORKSPACE, "dsa_indexer_topk_varlen: null or misaligned workspace");
  if (ws_bytes < dsa_indexer_topk_varlen_workspace(vl, H_I, d_I, k))
    return set_error(DSA_ERR_WORKSPACE, "dsa_indexer_topk_varlen: workspace too small");
  st = indexer_topk_launch(q_idx, k_idx, w, vl->B, vl->max_Lq, vl->max_Lk, 0, H_I, d_I, k, idx, ws, ws_bytes,
                           static_cast<cudaStream_t>(stream), &va);
  if (st == DSA_OK) g_indexer_launches.fetch_add(1);
  return st;
}

size_t dsa_sparse_attn_varlen_workspace(const dsa_varlen* vl, int n_h, int D_v, int k) {
  if (check_varlen_host(vl, nullptr) != DSA_OK || n_h < 1 || D_v < 1 || k < 1) return 0;
  return sparse_attn_ws_rows(vl->total_q, n_h, D_v, k);
}

dsa_status dsa_sparse_attn_varlen(const dsa_bf16* q, const dsa_bf16* kbuf, int64_t k_row_stride,
                                  const dsa_bf16* vbuf, int64_t v_row_stride, const int32_t* idx,
                                  const dsa_varlen* vl, int n_h, int D_qk, int D_v, int k, float scale,
                                  dsa_bf16* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
  VarlenArgs va{};
  dsa_status st = check_varlen_host(vl, &va);
  if (st != DSA_OK) return st;
  if (!q || !kbuf || !vbuf || !idx || !out)
    return set_error(DSA_ERR_INVALID_ARG, "dsa_sparse_attn_varlen: null pointer");
  if (!aligned16(q) || !aligned16(kbuf) || !aligned16(vbuf) || !aligned16(idx) || !aligned16(out) ||
      (lse && !aligned16(lse)))
    return set_error(DSA_ERR_INVALID_ARG, "dsa_sparse_attn_varlen: pointers must be 16-byte aligned");
  if (n_h < 1 || D_qk < 1 || D_v < 1 || k < 1)
    return set_error(DSA_ERR_INVALID_ARG, "dsa_sparse_attn_varlen: sizes must be positive");
  if (k_row_stride < D_qk || v_row_stride < D_v || (k_row_stride % 8) || (v_row_stride % 8))
    return set_error(DSA_ERR_INVALID_ARG, "dsa_sparse_attn_varlen: row strides must cover the row and be multiples of 8");
  return sparse_attn_launch(q, kbuf, k_row_stride, vbuf, v_row_stride, idx, vl->B, vl->max_Lq, vl->max_Lk, 0,
                            n_h, D_qk, D_v, k, scale, out, lse, ws, ws_bytes, static_cast<cudaStream_t>(stream),
                            &va);
}

size_t indexcache_forward_varlen_workspace(const dsa_dims* d, const dsa_varlen* vl) {
  if (!d) return 0;
  return std::max(dsa_indexer_topk_varlen_workspace(vl, d->H_I, d->d_I, d->k),
                  dsa_sparse_attn_varlen_workspace(vl, d->n_h, d->D_v, d->k));
}

dsa_status indexcache_forward_varlen(const char* pattern, int n_layers, const dsa_layer_io* layers,
                                     const dsa_dims* dims, const dsa_varlen* vl, int32_t* idx_cache, void* ws,
                                     size_t ws_bytes, void* stream) {
  // [IC] §1.1: the pattern rules of indexcache_forward
  if (!pattern || n_layers < 1) return set_error(DSA_ERR_BAD_PATTERN, "indexcache_forward_varlen: empty pattern");
  if (pattern[0] != 'F')
    return set_error(DSA_ERR_BAD_PATTERN, "indexcache_forward_varlen: the first layer must be 'F'");
  for (int l = 0; l < n_layers; ++l)
    if (pattern[l] != 'F' && pattern[l] != 'S')
      return set_error(DSA_ERR_BAD_PATTERN, "indexcache_forward_varlen: pattern entries must be 'F' or 'S'");
  if (!layers || !dims || !idx_cache)
    return set_error(DSA_ERR_INVALID_ARG, "indexcache_forward_varlen: null pointer");
  dsa_status st = check_varlen_host(vl, nullptr);
  if (st != DSA_OK) return st;
  const dsa_dims& d = *dims;
  if (ws_bytes < indexcache_forward_varlen_workspace(dims, vl))
    return set_error(DSA_ERR_WORKSPACE, "indexcache_forward_varlen: workspace too small");
  for (int l = 0; l < n_layers; ++l) {
    const dsa_layer_io& L = layers[l];
    if (pattern[l] == 'F') {
      st = check_indexer_args(L.q_idx, L.k_idx, L.w, 1, vl->max_Lq, vl->max_Lk, 0, d.H_I, d.d_I, d.k, idx_cache);
      if (st != DSA_OK) return st;
    }
    if (!L.q || !L.kbuf || !L.vbuf || !L.out)
      return set_error(DSA_ERR_INVALID_ARG, "indexcache_forward_varlen: null attention pointer");
  }
  // [IC] §1.2, Figure 2, per sequence of the batch
  for (int l = 0; l < n_layers; ++l) {
    const dsa_layer_io& L = layers[l];
    if (pattern[l] == 'F') {
      st = dsa_indexer_topk_varlen(L.q_idx, L.k_idx, L.w, vl, d.H_I, d.d_I, d.k, idx_cache, ws, ws_bytes, stream);
      if (st != DSA_OK) return st;
    }
    st = dsa_sparse_attn_varlen(L.q, L.kbuf, d.k_row_stride, L.vbuf, d.v_row_stride, idx_cache, vl, d.n_h, d.D_qk,
                                d.D_v, d.k, d.scale, L.out, L.lse, ws, ws_bytes, stream);
    if (st != DSA_OK) return st;
  }
  return DSA_OK;
}

dsa_status dsa_check_varlen(const dsa_varlen* vl, int* bad_seqs, void* stream) {
  dsa_status st = check_varlen_host(vl, nullptr);
  if (st != DSA_OK) return st;
  if (!bad_seqs) return set_error(DSA_ERR_INVALID_ARG, "dsa_check_varlen: null pointer");
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(bad_seqs, 0, sizeof(int), s);
  if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("dsa_check_varlen: ") + cudaGetErrorString(e));
  const unsigned blocks = static_cast<unsigned>(std::min(1024, (vl->B + 255) / 256));
  check_varlen_kernel<<<blocks, 256, 0, s>>>(vl->cu_q, vl->cu_k, vl->start_pos, vl->B, vl->total_q, vl->total_k,
                                             vl->max_Lq, vl->max_Lk, bad_seqs);
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("dsa_check_varlen launch: ") + cudaGetErrorString(e));
  return DSA_OK;
}

dsa_status dsa_check_indices(const int32_t* idx, int B, int Lq, int start_pos, int k, int* bad_rows,
                             void* stream) {
  if (!idx || !bad_rows) return set_error(DSA_ERR_INVALID_ARG, "dsa_check_indices: null pointer");
  if (B < 1 || Lq < 1 || k < 1 || start_pos < 0)
    return set_error(DSA_ERR_INVALID_ARG, "dsa_check_indices: sizes must be positive");
  const long long rows = static_cast<long long>(B) * Lq;
  if (rows > 2147483647ll) return set_error(DSA_ERR_UNSUPPORTED, "dsa_check_indices: too many rows");
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(bad_rows, 0, sizeof(int), st);
  if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("dsa_check_indices: ") + cudaGetErrorString(e));
  check_indices_kernel<<<static_cast<unsigned>(rows), 32, 0, st>>>(idx, Lq, start_pos, k, bad_rows);
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("dsa_check_indices launch: ") + cudaGetErrorString(e));
  return DSA_OK;
}

dsa_status dsa_selftest_wait_timeout(long long limit_cycles, void* stream) {
  if (limit_cycles < 1 || limit_cycles > 2000000000ll)
    return set_error(DSA_ERR_INVALID_ARG, "dsa_selftest_wait_timeout: limit out of range");
  unsigned int* err = device_error_word();
  if (!err) return set_error(DSA_ERR_CUDA, "cannot resolve the device error word");
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err, limit_cycles);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("self-test launch: ") + cudaGetErrorString(e));
  return DSA_OK;
}

dsa_status dsa_check_device_errors(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("stream sync: ") + cudaGetErrorString(e));
  unsigned int word = 0;
  e = cudaMemcpyFromSymbol(&word, g_dsa_error, sizeof(word));
  if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("read error word: ") + cudaGetErrorString(e));
  if (word) {
    const unsigned int zero = 0;
    cudaMemcpyToSymbol(g_dsa_error, &zero, sizeof(zero));
    return set_error(DSA_ERR_TIMEOUT, "a kernel's bounded wait expired");
  }
  return DSA_OK;
}

}  // extern "C"
