// lowprec.cu -- the low-precision selector of "注意力机制中的 Index" §5.4:
// the lightning-indexer score with the QK product on low-precision operands
// (FP8 E4M3 or FP4 E2M1) and the score quantised from fp32 to bf16 before the
// top-k.  The pages name the formats only; the element and scale rules are
// those of the OCP Microscaling (MX) v1.0 format that block-scaled tensor-core
// products consume: every 32 consecutive elements of a row share a power-of-
// two scale X = 2^(floor(log2 amax) - emax) (emax 8 for E4M3, 2 for E2M1),
// stored as an 8-bit exponent (ue8m0), and each element becomes the format
// value nearest to x / X (ties to even, saturating at the largest finite
// value).
//
// mx_quantize_kernel  one warp per row of 128 bf16 elements (4 blocks): block
//     maxima by warp shuffles, the exponent from the bit pattern of the
//     maximum, conversions by the hardware's round-to-nearest-even,
//     saturating cvt.  E4M3 codes are one byte per element; E2M1 codes are
//     packed two per byte, 16 codes in the first half of each 16-byte slot
//     (the layout the block-scaled MMA reads sub-byte operands in), so a row
//     takes 128 bytes either way.  Scales go
//     either row-major ([rows][4]) or grouped by 128 rows in the layout the
//     TMEM copy of the MMA kernel reads.
// The selector itself is the fused indexer + top-k kernel of indexer_topk.cu
// instantiated for MX operands.
#include <cuda_bf16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include <algorithm>
#include <cmath>

#include "dsa_internal.h"
#include "dsa_ptx.cuh"

namespace dsa {
namespace {

constexpr int kCols = 128;          // elements per row (d_I)
constexpr int kQuantThreads = 256;  // 8 rows per block

template <int FMT>  // 0: E4M3, 1: E2M1
__global__ void __launch_bounds__(kQuantThreads)
mx_quantize_kernel(const __nv_bfloat16* __restrict__ x, int B, long long rows_per_batch, int groups_per_batch,
                   int grouped, uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
  constexpr int kEmax = FMT == 0 ? 8 : 2;
  const int lane = threadIdx.x & 31;
  const long long padded = grouped ? static_cast<long long>(groups_per_batch) * 128 : rows_per_batch;
  const long long total = static_cast<long long>(B) * padded;
  const long long warps = static_cast<long long>(gridDim.x) * (kQuantThreads / 32);
  pdl_trigger();
  pdl_wait();
  for (long long gw = (static_cast<long long>(blockIdx.x) * kQuantThreads + threadIdx.x) >> 5; gw < total;
       gw += warps) {
    const long long b = gw / padded, r = gw % padded;
    const long long row = b * rows_per_batch + r;
    uint8_t* sfp = grouped ? sf + (b * groups_per_batch + r / 128) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4
                           : sf + row * 4;
    if (r >= rows_per_batch) {  // padding rows of the last group: unit scale
      if (lane < 4) sfp[lane] = 127;
      continue;
    }
    // lane l holds elements 4l .. 4l + 3, in block l / 8
    const uint2 raw = __ldg(reinterpret_cast<const uint2*>(x + row * kCols) + lane);
    float v[4];
    v[0] = __uint_as_float(raw.x << 16);
    v[1] = __uint_as_float(raw.x & 0xFFFF0000u);
    v[2] = __uint_as_float(raw.y << 16);
    v[3] = __uint_as_float(raw.y & 0xFFFF0000u);
    float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    // X = 2^(floor(log2 amax) - emax); an all-zero block takes 2^-emax
    const int e = (amax > 0.f ? ilogbf(amax) : 0) - kEmax;
    uint32_t packed;
    if constexpr (FMT == 0) {
      const __nv_fp8x2_storage_t lo =
          __nv_cvt_float2_to_fp8x2(make_float2(ldexpf(v[0], -e), ldexpf(v[1], -e)), __NV_SATFINITE, __NV_E4M3);
      const __nv_fp8x2_storage_t hi =
          __nv_cvt_float2_to_fp8x2(make_float2(ldexpf(v[2], -e), ldexpf(v[3], -e)), __NV_SATFINITE, __NV_E4M3);
      packed = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
    } else {
      // two codes per byte, the even element in the low nibble
      const __nv_fp4x2_storage_t lo =
          __nv_cvt_float2_to_fp4x2(make_float2(ldexpf(v[0], -e), ldexpf(v[1], -e)), __NV_E2M1, cudaRoundNearest);
      const __nv_fp4x2_storage_t hi =
          __nv_cvt_float2_to_fp4x2(make_float2(ldexpf(v[2], -e), ldexpf(v[3], -e)), __NV_E2M1, cudaRoundNearest);
      const uint32_t mine = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 8);
      // The block-scaled MMA reads sub-byte operands as 16 codes packed in
      // the first 8 bytes of each 16-byte slot (the rest zero): word l of
      // the row is slot l / 4, quarter q = l % 4; quarters 0 and 1 hold the
      // slot's codes 0-7 and 8-15, i.e. the 16-bit pieces of lanes
      // 4 (l / 4) + 2 q and the next one.
      const int q = lane & 3;
      const int src = (lane & ~3) + 2 * (q & 1);
      const uint32_t a = __shfl_sync(0xffffffffu, mine, src);
      const uint32_t b2 = __shfl_sync(0xffffffffu, mine, src + 1);
      packed = q < 2 ? (a | (b2 << 16)) : 0u;
    }
    reinterpret_cast<uint32_t*>(codes + row * kCols)[lane] = packed;
    if ((lane & 7) == 0) sfp[lane >> 3] = static_cast<uint8_t>(min(max(e + 127, 0), 254));
  }
}

dsa_status quantize_launch(const dsa_bf16* x, int B, long long rows_per_batch, int groups_per_batch, bool grouped,
                           int fmt, uint8_t* codes, uint8_t* sf, cudaStream_t stream) {
  const long long padded = grouped ? static_cast<long long>(groups_per_batch) * 128 : rows_per_batch;
  const long long warps = static_cast<long long>(B) * padded;
  const int sms = device_sm_count();
  if (sms <= 0) return set_error(DSA_ERR_CUDA, "cannot query the device SM count");
  const unsigned blocks =
      static_cast<unsigned>(std::max<long long>(1, std::min<long long>((warps + 7) / 8, 16ll * sms)));
  const auto* xb = reinterpret_cast<const __nv_bfloat16*>(x);
  cudaError_t e = fmt == DSA_FMT_E4M3
                      ? launch_pdl(mx_quantize_kernel<0>, dim3(blocks), dim3(kQuantThreads), 0, stream, xb, B,
                                   rows_per_batch, groups_per_batch, static_cast<int>(grouped), codes, sf)
                      : launch_pdl(mx_quantize_kernel<1>, dim3(blocks), dim3(kQuantThreads), 0, stream, xb, B,
                                   rows_per_batch, groups_per_batch, static_cast<int>(grouped), codes, sf);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("quantize launch: ") + cudaGetErrorString(e));
  return DSA_OK;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Workspace layout of the selector: the indexer plan's buffers, then the
// query codes and scales, then the key codes and scales.
struct LowprecLayout {
  size_t plan, codes_q, sf_q, codes_k, sf_k, total;
  int sfq_groups, sfk_tiles;
};

LowprecLayout lowprec_layout(int B, int Lq, int Lk, int start_pos, int k) {
  LowprecLayout l{};
  l.plan = align256(indexer_plan(B, Lq, Lk, start_pos, std::min(k, 2048)).total_bytes);
  l.sfq_groups = (Lq + 7) / 8 * 4;  // 4 groups of 128 (query, head) rows per 8-query block
  l.sfk_tiles = (Lk + 127) / 128;
  l.codes_q = align256(static_cast<size_t>(B) * Lq * 64 * kCols);
  l.sf_q = align256(static_cast<size_t>(B) * l.sfq_groups * 512);
  l.codes_k = align256(static_cast<size_t>(B) * Lk * kCols);
  l.sf_k = align256(static_cast<size_t>(B) * l.sfk_tiles * 512);
  l.total = l.plan + l.codes_q + l.sf_q + l.codes_k + l.sf_k;
  return l;
}

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" {

dsa_status dsa_mx_quantize(const dsa_bf16* x, int64_t rows, int cols, int fmt, uint8_t* codes, uint8_t* scales,
                           void* stream) {
  if (!x || !codes || !scales) return set_error(DSA_ERR_INVALID_ARG, "dsa_mx_quantize: null pointer");
  if (!aligned16(x) || !aligned16(codes)) return set_error(DSA_ERR_INVALID_ARG, "dsa_mx_quantize: pointers must be 16-byte aligned");
  if (rows < 1) return set_error(DSA_ERR_INVALID_ARG, "dsa_mx_quantize: rows must be positive");
  if (cols != kCols) return set_error(DSA_ERR_UNSUPPORTED, "dsa_mx_quantize: rows of 128 elements");
  if (fmt != DSA_FMT_E4M3 && fmt != DSA_FMT_E2M1) return set_error(DSA_ERR_INVALID_ARG, "dsa_mx_quantize: unknown format");
  return quantize_launch(x, 1, rows, 0, false, fmt, codes, scales, static_cast<cudaStream_t>(stream));
}

size_t dsa_indexer_topk_lowprec_workspace(int B, int Lq, int Lk, int start_pos, int H_I, int d_I, int k, int fmt) {
  if (B < 1 || Lq < 1 || Lk < 1 || start_pos < 0 || k < 1 || H_I != 64 || d_I != kCols) return 0;
  if (fmt != DSA_FMT_E4M3 && fmt != DSA_FMT_E2M1) return 0;
  return lowprec_layout(B, Lq, Lk, start_pos, k).total;
}

dsa_status dsa_indexer_topk_lowprec(const dsa_bf16* q_idx, const dsa_bf16* k_idx, const float* w, int B, int Lq,
                                    int Lk, int start_pos, int H_I, int d_I, int k, int fmt, int32_t* idx, void* ws,
                                    size_t ws_bytes, void* stream) {
  if (!q_idx || !k_idx || !w || !idx) return set_error(DSA_ERR_INVALID_ARG, "dsa_indexer_topk_lowprec: null pointer");
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w) || !aligned16(idx))
    return set_error(DSA_ERR_INVALID_ARG, "dsa_indexer_topk_lowprec: pointers must be 16-byte aligned");
  if (B < 1 || Lq < 1 || Lk < 1 || start_pos < 0 || k < 1)
    return set_error(DSA_ERR_INVALID_ARG, "dsa_indexer_topk_lowprec: sizes must be positive");
  if (static_cast<long long>(start_pos) + Lq - 1 > Lk)
    return set_error(DSA_ERR_INVALID_ARG, "dsa_indexer_topk_lowprec: start_pos + Lq - 1 exceeds Lk");
  if (fmt != DSA_FMT_E4M3 && fmt != DSA_FMT_E2M1)
    return set_error(DSA_ERR_INVALID_ARG, "dsa_indexer_topk_lowprec: unknown format");
  if (H_I != 64 || d_I != kCols || k > 2048)
    return set_error(DSA_ERR_UNSUPPORTED, "dsa_indexer_topk_lowprec: H_I = 64, d_I = 128, k <= 2048");
  if (static_cast<long long>(Lq) * H_I > (1ll << 31) - 1 || static_cast<long long>(B) * Lq * k > (1ll << 40))
    return set_error(DSA_ERR_UNSUPPORTED, "dsa_indexer_topk_lowprec: tensor too large");
  if (!ws || !aligned16(ws)) return set_error(DSA_ERR_WORKSPACE, "dsa_indexer_topk_lowprec: null or misaligned workspace");
  const LowprecLayout l = lowprec_layout(B, Lq, Lk, start_pos, k);
  if (ws_bytes < l.total) return set_error(DSA_ERR_WORKSPACE, "dsa_indexer_topk_lowprec: workspace too small");
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint8_t* codes_q = base + l.plan;
  uint8_t* sf_q = codes_q + l.codes_q;
  uint8_t* codes_k = sf_q + l.sf_q;
  uint8_t* sf_k = codes_k + l.codes_k;
  // query rows are (query, head) pairs: 64 per query
  dsa_status st = quantize_launch(q_idx, B, static_cast<long long>(Lq) * 64, l.sfq_groups, true, fmt, codes_q, sf_q, s);
  if (st != DSA_OK) return st;
  st = quantize_launch(k_idx, B, Lk, l.sfk_tiles, true, fmt, codes_k, sf_k, s);
  if (st != DSA_OK) return st;
  return indexer_topk_mx_launch(codes_q, codes_k, sf_q, sf_k, l.sfq_groups, l.sfk_tiles, w, B, Lq, Lk, start_pos,
                                fmt == DSA_FMT_E4M3 ? 0 : 5, k, idx, ws, l.plan, s);
}

}  // extern "C"
