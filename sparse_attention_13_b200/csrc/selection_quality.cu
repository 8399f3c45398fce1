// selection_quality.cu -- measurement tools for index selections, after
// [IDX] "注意力机制中的 Index：从位置下标到预算检索" §8 (how index quality is
// evaluated):
//   - dense_weights_kernel: the dense attention weights alpha^dense_{t,s}
//     that a selection is scored against (§8.1), averaged over heads, and the
//     dense log-sum-exp per head;
//   - topk_rows_kernel: TopK_k over a dense row of scores (§8.2's oracle
//     selection), in the library's row form (ascending s, then -1);
//   - index_overlap_kernel: |A & B| per row, the numerator of Recall@k (§8.2)
//     and of the adjacent-layer overlap (§8.4);
//   - captured_mass_kernel: CapturedMass@k (§8.1) as exp(lse_S - lse_{P_t}).
// They measure selections on short contexts and are not on the layer loop's
// path, so they are plain CUDA-core kernels, one CTA per row.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <algorithm>
#include <string>

#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr int kDwThreads = 256;  // 16 head groups x 16 key groups
constexpr int kDwHeads = 128;    // head slots: head h = hg + 16 i, i < 8
constexpr int kDwKeys = 64;      // keys per tile: key r = kg + 16 j, j < 4
constexpr int kDwMaxD = 576;

// Shared-memory row pitch in 32-bit words: D/2 + 1 is odd for D % 4 == 0, so
// 16 consecutive rows start in 16 different banks.
__host__ __device__ constexpr int dw_pitch(int D) { return D / 2 + 1; }
__host__ __device__ constexpr int dw_smem_bytes(int D) {
  return (kDwHeads + kDwKeys) * dw_pitch(D) * 4 + (kDwThreads / 32) * kDwKeys * 4;
}

__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// Copies `rows` rows of D bf16 (16-byte aligned, D % 8 == 0) into smem at the
// odd pitch; rows at or past `valid` are zero-filled.
__device__ __forceinline__ void dw_load_rows(uint32_t* dst, const dsa_bf16* src, int64_t stride,
                                             int rows, int valid, int D) {
  const int per_row = D / 8;
  const int pitch = dw_pitch(D);
  for (int e = threadIdx.x; e < rows * per_row; e += kDwThreads) {
    const int r = e / per_row, c = e % per_row;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (r < valid) v = *reinterpret_cast<const uint4*>(src + r * stride + c * 8);
    uint32_t* d = dst + r * pitch + c * 4;
    d[0] = v.x;
    d[1] = v.y;
    d[2] = v.z;
    d[3] = v.w;
  }
}

// acc[i][j] = q[hg + 16 i] . K[kg + 16 j] over D columns, in fp32 with a fixed
// order (both passes of dense_weights_kernel get identical dots).
__device__ __forceinline__ void dw_dots(const uint32_t* sq, const uint32_t* sk, int D, int hg, int kg,
                                        float (&acc)[8][4]) {
  const int pitch = dw_pitch(D);
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  const uint32_t* qb = sq + hg * pitch;
  const uint32_t* kb = sk + kg * pitch;
#pragma unroll 2
  for (int c = 0; c < D / 2; ++c) {
    uint32_t qu[8], ku[4];
#pragma unroll
    for (int i = 0; i < 8; ++i) qu[i] = qb[16 * i * pitch + c];
#pragma unroll
    for (int j = 0; j < 4; ++j) ku[j] = kb[16 * j * pitch + c];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        acc[i][j] = fmaf(bf_lo(qu[i]), bf_lo(ku[j]), acc[i][j]);
        acc[i][j] = fmaf(bf_hi(qu[i]), bf_hi(ku[j]), acc[i][j]);
      }
  }
}

// One CTA per query row (longest rows first).  Pass 1: per head, the running
// max and sum of exp(scale * q.K[s]) over s < t, combined across the 16 key
// groups: lse[h].  Pass 2 (mean_w != nullptr): mean_w[s] = (1/n_h) sum_h
// exp(scale * q.K[s] - lse[h]) for s < t.
__global__ void __launch_bounds__(kDwThreads, 1)
    dense_weights_kernel(const dsa_bf16* __restrict__ q, const dsa_bf16* __restrict__ kbuf,
                         int64_t k_stride, int B, int Lq, int Lk, int start_pos, int n_h, int D,
                         float scale, float* __restrict__ lse_out, float* __restrict__ mean_w) {
  extern __shared__ __align__(16) uint32_t dw_smem[];
  uint32_t* sq = dw_smem;
  uint32_t* sk = sq + kDwHeads * dw_pitch(D);
  float* red = reinterpret_cast<float*>(sk + kDwKeys * dw_pitch(D));

  const int b = blockIdx.x % B;
  const int i = Lq - 1 - static_cast<int>(blockIdx.x / B);
  const int T = start_pos + i;
  const int64_t row = static_cast<int64_t>(b) * Lq + i;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int hg = tid >> 4, kg = tid & 15;
  const dsa_bf16* krow0 = kbuf + static_cast<int64_t>(b) * Lk * k_stride;

  dw_load_rows(sq, q + row * n_h * D, D, kDwHeads, n_h, D);

  float m[8], z[8];
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    m[a] = -INFINITY;
    z[a] = 0.f;
  }
  float acc[8][4];
  for (int s0 = 0; s0 < T; s0 += kDwKeys) {
    __syncthreads();
    dw_load_rows(sk, krow0 + s0 * k_stride, k_stride, kDwKeys, min(kDwKeys, T - s0), D);
    __syncthreads();
    dw_dots(sq, sk, D, hg, kg, acc);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (s0 + kg + 16 * j >= T) continue;
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        const float e = scale * acc[a][j];
        if (e > m[a]) {
          z[a] = z[a] * expf(m[a] - e) + 1.f;
          m[a] = e;
        } else {
          z[a] += expf(e - m[a]);
        }
      }
    }
  }
  // combine the 16 key groups (lanes of one half-warp share hg)
  float lse[8];
#pragma unroll
  for (int a = 0; a < 8; ++a) {
#pragma unroll
    for (int off = 8; off >= 1; off >>= 1) {
      const float mo = __shfl_xor_sync(0xffffffffu, m[a], off);
      const float zo = __shfl_xor_sync(0xffffffffu, z[a], off);
      const float mn = fmaxf(m[a], mo);
      z[a] = mn == -INFINITY ? 0.f : z[a] * expf(m[a] - mn) + zo * expf(mo - mn);
      m[a] = mn;
    }
    lse[a] = z[a] > 0.f ? m[a] + logf(z[a]) : -INFINITY;
    const int h = hg + 16 * a;
    if (kg == 0 && h < n_h) lse_out[row * n_h + h] = lse[a];
  }
  if (mean_w == nullptr) return;

  const float inv_nh = 1.f / static_cast<float>(n_h);
  float* wrow = mean_w + row * Lk;
  for (int s0 = 0; s0 < T; s0 += kDwKeys) {
    __syncthreads();
    dw_load_rows(sk, krow0 + s0 * k_stride, k_stride, kDwKeys, min(kDwKeys, T - s0), D);
    __syncthreads();
    dw_dots(sq, sk, D, hg, kg, acc);
    float part[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      part[j] = 0.f;
#pragma unroll
      for (int a = 0; a < 8; ++a)
        if (hg + 16 * a < n_h) part[j] += expf(scale * acc[a][j] - lse[a]);
      part[j] += __shfl_xor_sync(0xffffffffu, part[j], 16);
      if (lane < 16) red[warp * kDwKeys + kg + 16 * j] = part[j];
    }
    __syncthreads();
    if (tid < kDwKeys && s0 + tid < T) {
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kDwThreads / 32; ++w) sum += red[w * kDwKeys + tid];
      wrow[s0 + tid] = sum * inv_nh;
    }
  }
}

constexpr int kTkThreads = 512;

// Order-preserving map of a finite float onto uint32 (-0 counts as +0).
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f == 0.f ? 0.f : f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// One CTA per row: TopK_k over the t = start_pos + (row % Lq) leading scores,
// ties to the lower position, written ascending and padded with -1.  Four
// 8-bit radix passes find the k-th largest key and how many of its ties are
// taken; one ordered pass then writes the selection.
__global__ void __launch_bounds__(kTkThreads)
    topk_rows_kernel(const float* __restrict__ scores, int64_t ld, int Lq, int start_pos, int k,
                     int32_t* __restrict__ idx) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t warp_tot[kTkThreads / 32];
  __shared__ uint32_t s_prefix, s_need;
  const int64_t row = blockIdx.x;
  const int T = start_pos + static_cast<int>(row % Lq);
  const float* sr = scores + row * ld;
  int32_t* out = idx + row * k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (T <= k) {
    for (int e = tid; e < k; e += kTkThreads) out[e] = e < T ? e : -1;
    return;
  }
  uint32_t prefix = 0, mask = 0, need = static_cast<uint32_t>(k);
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int d = tid; d < 256; d += kTkThreads) hist[d] = 0;
    __syncthreads();
    for (int s = tid; s < T; s += kTkThreads) {
      const uint32_t key = order_key(sr[s]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      uint32_t cum = 0;
      int d = 255;
      for (; d > 0; --d) {
        if (cum + hist[d] >= need) break;
        cum += hist[d];
      }
      s_prefix = prefix | (static_cast<uint32_t>(d) << shift);
      s_need = need - cum;
    }
    __syncthreads();
    prefix = s_prefix;
    need = s_need;
    mask |= 255u << shift;
  }
  // prefix is the k-th largest key; `need` of its ties are taken, lowest
  // positions first.  Counts per 512-position chunk fit in 16 bits.
  uint32_t gt_base = 0, tie_base = 0;
  for (int base = 0; base < T; base += kTkThreads) {
    const int s = base + tid;
    const uint32_t key = s < T ? order_key(sr[s]) : 0u;
    const uint32_t gt = (s < T && key > prefix) ? 1u : 0u;
    const uint32_t tie = (s < T && key == prefix) ? 1u : 0u;
    const uint32_t v = (gt << 16) | tie;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    uint32_t before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kTkThreads / 32; ++w) {
      const uint32_t c = warp_tot[w];
      if (w < warp) before += c;
      total += c;
    }
    const uint32_t excl = before + x - v;
    const uint32_t gt_before = gt_base + (excl >> 16);
    const uint32_t tie_before = tie_base + (excl & 0xffffu);
    if (gt || (tie && tie_before < need)) out[gt_before + min(tie_before, need)] = s;
    gt_base += total >> 16;
    tie_base += total & 0xffffu;
    __syncthreads();
  }
}

constexpr int kOvThreads = 256;

// |A & B| for one pair of rows in the library's row form (ascending, then
// -1): each valid entry of A is looked up in B by binary search, with -1
// ordered after every position.
__global__ void __launch_bounds__(kOvThreads)
    index_overlap_kernel(const int32_t* __restrict__ a, const int32_t* __restrict__ b, int k,
                         int32_t* __restrict__ inter) {
  __shared__ int warp_cnt[kOvThreads / 32];
  const int64_t row = blockIdx.x;
  const int32_t* ar = a + row * k;
  const int32_t* br = b + row * k;
  int cnt = 0;
  for (int e = threadIdx.x; e < k; e += kOvThreads) {
    const int32_t v = ar[e];
    if (v < 0) continue;
    int lo = 0, hi = k;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      const int32_t x = br[mid];
      const uint32_t kx = x < 0 ? 0xffffffffu : static_cast<uint32_t>(x);
      if (kx < static_cast<uint32_t>(v))
        lo = mid + 1;
      else
        hi = mid;
    }
    cnt += (lo < k && br[lo] == v) ? 1 : 0;
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if ((threadIdx.x & 31) == 0) warp_cnt[threadIdx.x >> 5] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    int total = 0;
#pragma unroll
    for (int w = 0; w < kOvThreads / 32; ++w) total += warp_cnt[w];
    inter[row] = total;
  }
}

// CapturedMass = exp(lse_S - lse_{P_t}); a row that sees nothing has mass 1.
__global__ void captured_mass_kernel(const float* __restrict__ lse_sel, const float* __restrict__ lse_dense,
                                     int64_t n, float* __restrict__ mass) {
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float d = lse_dense[e];
    mass[e] = d == -INFINITY ? 1.f : expf(lse_sel[e] - d);
  }
}

dsa_status launch_status(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
  return DSA_OK;
}

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" {

dsa_status dsa_dense_weights(const dsa_bf16* q, const dsa_bf16* kbuf, int64_t k_row_stride, int B,
                             int Lq, int Lk, int start_pos, int n_h, int D_qk, float scale,
                             float* lse_dense, float* mean_w, void* stream) {
  if (!q || !kbuf || !lse_dense) return set_error(DSA_ERR_INVALID_ARG, "dsa_dense_weights: null pointer");
  if (!aligned16(q) || !aligned16(kbuf))
    return set_error(DSA_ERR_INVALID_ARG, "dsa_dense_weights: pointers must be 16-byte aligned");
  if (B < 1 || Lq < 1 || Lk < 1 || start_pos < 0 || n_h < 1 || D_qk < 1)
    return set_error(DSA_ERR_INVALID_ARG, "dsa_dense_weights: sizes must be positive");
  if (static_cast<long long>(start_pos) + Lq - 1 > Lk)
    return set_error(DSA_ERR_INVALID_ARG, "dsa_dense_weights: start_pos + Lq - 1 exceeds Lk");
  if (n_h > kDwHeads || D_qk > kDwMaxD || D_qk % 8 != 0)
    return set_error(DSA_ERR_UNSUPPORTED, "dsa_dense_weights: needs n_h <= 128 and D_qk <= 576, a multiple of 8");
  if (k_row_stride < D_qk || k_row_stride % 8 != 0)
    return set_error(DSA_ERR_INVALID_ARG, "dsa_dense_weights: k_row_stride must cover the row and be a multiple of 8");
  if (static_cast<long long>(B) * Lq > 2147483647ll)
    return set_error(DSA_ERR_UNSUPPORTED, "dsa_dense_weights: too many rows");
  const int smem = dw_smem_bytes(D_qk);
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(dense_weights_kernel), smem);
  if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("dsa_dense_weights: ") + cudaGetErrorString(e));
  dense_weights_kernel<<<static_cast<unsigned>(B * Lq), kDwThreads, smem, static_cast<cudaStream_t>(stream)>>>(
      q, kbuf, k_row_stride, B, Lq, Lk, start_pos, n_h, D_qk, scale, lse_dense, mean_w);
  return launch_status("dsa_dense_weights launch");
}

dsa_status dsa_topk_rows(const float* scores, int64_t row_stride, int B, int Lq, int start_pos, int k,
                         int32_t* idx, void* stream) {
  if (!scores || !idx) return set_error(DSA_ERR_INVALID_ARG, "dsa_topk_rows: null pointer");
  if (B < 1 || Lq < 1 || k < 1 || start_pos < 0 || row_stride < 1)
    return set_error(DSA_ERR_INVALID_ARG, "dsa_topk_rows: sizes must be positive");
  if (static_cast<long long>(start_pos) + Lq - 1 > row_stride)
    return set_error(DSA_ERR_INVALID_ARG, "dsa_topk_rows: start_pos + Lq - 1 exceeds row_stride");
  if (static_cast<long long>(B) * Lq > 2147483647ll)
    return set_error(DSA_ERR_UNSUPPORTED, "dsa_topk_rows: too many rows");
  topk_rows_kernel<<<static_cast<unsigned>(B * Lq), kTkThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      scores, row_stride, Lq, start_pos, k, idx);
  return launch_status("dsa_topk_rows launch");
}

dsa_status dsa_index_overlap(const int32_t* a, const int32_t* b, int64_t rows, int k, int32_t* inter,
                             void* stream) {
  if (!a || !b || !inter) return set_error(DSA_ERR_INVALID_ARG, "dsa_index_overlap: null pointer");
  if (rows < 1 || k < 1) return set_error(DSA_ERR_INVALID_ARG, "dsa_index_overlap: sizes must be positive");
  if (rows > 2147483647ll) return set_error(DSA_ERR_UNSUPPORTED, "dsa_index_overlap: too many rows");
  index_overlap_kernel<<<static_cast<unsigned>(rows), kOvThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      a, b, k, inter);
  return launch_status("dsa_index_overlap launch");
}

dsa_status dsa_captured_mass(const float* lse_sel, const float* lse_dense, int64_t n, float* mass,
                             void* stream) {
  if (!lse_sel || !lse_dense || !mass) return set_error(DSA_ERR_INVALID_ARG, "dsa_captured_mass: null pointer");
  if (n < 1) return set_error(DSA_ERR_INVALID_ARG, "dsa_captured_mass: n must be positive");
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, 4L * device_sm_count());
  captured_mass_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      lse_sel, lse_dense, n, mass);
  return launch_status("dsa_captured_mass launch");
}

}  // extern "C"
