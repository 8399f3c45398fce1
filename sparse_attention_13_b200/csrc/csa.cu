// csa.cu -- the CSA-style indexer and attention over compressed blocks,
// [IDX] "注意力机制中的 Index：从位置下标到预算检索" §5.2: query t scores the
// compressed blocks s < floor(t/m) with the lightning-indexer score, keeps
// TopK_k of them, and the main attention reads the selected compressed
// entries as shared keys and values.
//
// The indexer reuses the fused indexer + top-k kernels.  Grouping the query
// rows by phase p = t mod m turns the floor rule into the ordinary causal
// rule: with start_pos = c*m, row j of phase p sits at t = c*m + p + m*j and
// sees floor(t/m) = c + j blocks.  The m phases of a sequence therefore run
// as m sequences of one launch (start c, ceil(Lq/m) rows each, the same
// compressed keys); copy kernels build the phase-major inputs and put the
// index rows back in token order.  One query row (decode) needs no regrouping.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <string>

#include "dsa_internal.h"

namespace dsa {
namespace {

// Row maps of the regrouping copies: dst row r <- src row src_row(r), or
// zeros where there is none (the padding rows of a short phase).
enum : int { kPhaseRows = 0, kReplicateKeys = 1, kTokenRows = 2 };

struct RowMap {
  int mode;
  int Lq, Lq2, m, N;  // query rows, rows per phase, phases, compressed blocks
};

__device__ __forceinline__ int64_t src_row(const RowMap& p, int64_t r) {
  if (p.mode == kPhaseRows) {  // (b*m + ph)*Lq2 + j  <-  b*Lq + ph + m*j
    const int64_t bp = r / p.Lq2;
    const int64_t j = r % p.Lq2;
    const int64_t i = bp % p.m + p.m * j;
    return i < p.Lq ? (bp / p.m) * p.Lq + i : -1;
  }
  if (p.mode == kReplicateKeys) {  // (b*m + ph)*N + s  <-  b*N + s
    const int64_t bp = r / p.N;
    return (bp / p.m) * p.N + r % p.N;
  }
  // kTokenRows: b*Lq + i  <-  (b*m + i mod m)*Lq2 + floor(i/m)
  const int64_t b = r / p.Lq;
  const int64_t i = r % p.Lq;
  return (b * p.m + i % p.m) * p.Lq2 + i / p.m;
}

template <typename V>
__global__ void row_map_kernel(V* __restrict__ dst, const V* __restrict__ src, int64_t n_rows, int row_vecs,
                               const RowMap p) {
  const int64_t total = n_rows * row_vecs;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = e / row_vecs;
    const int c = static_cast<int>(e % row_vecs);
    const int64_t sr = src_row(p, r);
    V v{};
    if (sr >= 0) v = src[sr * row_vecs + c];
    dst[e] = v;
  }
}

dsa_status row_map(void* dst, const void* src, int64_t n_rows, int64_t row_bytes, const RowMap& p,
                   cudaStream_t stream) {
  const int sms = device_sm_count();
  if (sms <= 0) return set_error(DSA_ERR_CUDA, "cannot query the device SM count");
  const bool wide = row_bytes % 16 == 0 && aligned16(dst) && aligned16(src);
  const int64_t vec = wide ? 16 : 4;
  const int64_t row_vecs = row_bytes / vec;
  const int64_t total = n_rows * row_vecs;
  const unsigned blocks = static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>((total + 255) / 256, 8ll * sms)));
  if (wide)
    row_map_kernel<uint4><<<blocks, 256, 0, stream>>>(static_cast<uint4*>(dst), static_cast<const uint4*>(src),
                                                       n_rows, static_cast<int>(row_vecs), p);
  else
    row_map_kernel<uint32_t><<<blocks, 256, 0, stream>>>(static_cast<uint32_t*>(dst),
                                                          static_cast<const uint32_t*>(src), n_rows,
                                                          static_cast<int>(row_vecs), p);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("csa regrouping copy: ") + cudaGetErrorString(e));
  return DSA_OK;
}

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Workspace of the regrouped launch: phase-major q_idx, w, replicated keys,
// phase-major index rows, then the indexer's own workspace.
struct CsaPlan {
  bool direct;      // one launch of the token indexer on the given rows
  int start;        // start position of that launch (in blocks)
  int Lq2, B2;      // regrouped: rows per phase, sequences
  size_t q_off, w_off, k_off, i_off, ws_off, total;
};

CsaPlan csa_plan(int B, int Lq, int N, int start_pos, int m, int H, int d, int k) {
  CsaPlan pl{};
  if (Lq == 1 || m == 1) {
    pl.direct = true;
    pl.start = start_pos / m;
    pl.total = dsa_indexer_topk_workspace(B, Lq, N, pl.start, H, d, k);
    return pl;
  }
  pl.start = start_pos / m;
  pl.Lq2 = (Lq + m - 1) / m;
  pl.B2 = B * m;
  const size_t rows2 = static_cast<size_t>(pl.B2) * pl.Lq2;
  pl.q_off = 0;
  pl.w_off = align_up(pl.q_off + rows2 * H * d * 2);
  pl.k_off = align_up(pl.w_off + rows2 * H * 4);
  pl.i_off = align_up(pl.k_off + static_cast<size_t>(pl.B2) * N * d * 2);
  pl.ws_off = align_up(pl.i_off + rows2 * k * 4);
  pl.total = pl.ws_off + dsa_indexer_topk_workspace(pl.B2, pl.Lq2, N, pl.start, H, d, k);
  return pl;
}

// Shared checks: sizes, and that the last row's visible blocks exist.
dsa_status check_csa_shape(const char* who, int B, int Lq, int N, int start_pos, int m, int k) {
  if (B < 1 || Lq < 1 || N < 1 || start_pos < 0 || m < 1 || k < 1)
    return set_error(DSA_ERR_INVALID_ARG, std::string(who) + ": sizes must be positive");
  if ((static_cast<long long>(start_pos) + Lq - 1) / m > N)
    return set_error(DSA_ERR_INVALID_ARG, std::string(who) + ": floor((start_pos + Lq - 1) / m) exceeds N_cmp");
  return DSA_OK;
}

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" {

size_t dsa_csa_indexer_topk_workspace(int B, int Lq, int N_cmp, int start_pos, int m, int H_I, int d_I, int k) {
  if (B < 1 || Lq < 1 || N_cmp < 1 || start_pos < 0 || m < 1 || k < 1) return 0;
  if (static_cast<long long>(B) * m > 2147483647ll) return 0;
  return csa_plan(B, Lq, N_cmp, start_pos, m, H_I, d_I, k).total;
}

dsa_status dsa_csa_indexer_topk(const dsa_bf16* q_idx, const dsa_bf16* k_cmp, const float* w, int B, int Lq,
                                int N_cmp, int start_pos, int m, int H_I, int d_I, int k, int32_t* idx, void* ws,
                                size_t ws_bytes, void* stream) {
  if (!q_idx || !k_cmp || !w || !idx) return set_error(DSA_ERR_INVALID_ARG, "dsa_csa_indexer_topk: null pointer");
  dsa_status st = check_csa_shape("dsa_csa_indexer_topk", B, Lq, N_cmp, start_pos, m, k);
  if (st != DSA_OK) return st;
  if (Lq > 1 && m > 1 && start_pos % m != 0)
    return set_error(DSA_ERR_UNSUPPORTED, "dsa_csa_indexer_topk: several query rows need start_pos to be a multiple of m");
  if (static_cast<long long>(B) * m > 2147483647ll)
    return set_error(DSA_ERR_UNSUPPORTED, "dsa_csa_indexer_topk: too many sequences");
  const CsaPlan pl = csa_plan(B, Lq, N_cmp, start_pos, m, H_I, d_I, k);
  if (pl.direct)
    return dsa_indexer_topk(q_idx, k_cmp, w, B, Lq, N_cmp, pl.start, H_I, d_I, k, idx, ws, ws_bytes, stream);
  if (!indexer_supported(H_I, d_I, k))
    return set_error(DSA_ERR_UNSUPPORTED, "dsa_csa_indexer_topk: need H_I in {4,8,16,32,64}, d_I in {32,64,128}, k <= 2048");
  if (!aligned16(q_idx) || !aligned16(k_cmp) || !aligned16(w) || !aligned16(idx))
    return set_error(DSA_ERR_INVALID_ARG, "dsa_csa_indexer_topk: pointers must be 16-byte aligned");
  if (!ws || !aligned16(ws) || ws_bytes < pl.total)
    return set_error(DSA_ERR_WORKSPACE, "dsa_csa_indexer_topk: workspace too small");
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(ws);
  RowMap rm{kPhaseRows, Lq, pl.Lq2, m, N_cmp};
  const int64_t rows2 = static_cast<int64_t>(pl.B2) * pl.Lq2;
  st = row_map(base + pl.q_off, q_idx, rows2, static_cast<int64_t>(H_I) * d_I * 2, rm, s);
  if (st == DSA_OK) st = row_map(base + pl.w_off, w, rows2, static_cast<int64_t>(H_I) * 4, rm, s);
  rm.mode = kReplicateKeys;
  if (st == DSA_OK)
    st = row_map(base + pl.k_off, k_cmp, static_cast<int64_t>(pl.B2) * N_cmp, static_cast<int64_t>(d_I) * 2, rm, s);
  if (st != DSA_OK) return st;
  st = dsa_indexer_topk(reinterpret_cast<const dsa_bf16*>(base + pl.q_off),
                        reinterpret_cast<const dsa_bf16*>(base + pl.k_off),
                        reinterpret_cast<const float*>(base + pl.w_off), pl.B2, pl.Lq2, N_cmp, pl.start, H_I,
                        d_I, k, reinterpret_cast<int32_t*>(base + pl.i_off), base + pl.ws_off,
                        ws_bytes - pl.ws_off, stream);
  if (st != DSA_OK) return st;
  rm.mode = kTokenRows;
  return row_map(idx, base + pl.i_off, static_cast<int64_t>(B) * Lq, static_cast<int64_t>(k) * 4, rm, s);
}

dsa_status dsa_csa_sparse_attn(const dsa_bf16* q, const dsa_bf16* c_cmp, int64_t row_stride, const int32_t* idx,
                               int B, int Lq, int N_cmp, int start_pos, int m, int n_h, int D_qk, int D_v, int k,
                               float scale, dsa_bf16* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
  if (!q || !c_cmp || !idx || !out) return set_error(DSA_ERR_INVALID_ARG, "dsa_csa_sparse_attn: null pointer");
  if (!aligned16(q) || !aligned16(c_cmp) || !aligned16(idx) || !aligned16(out) || (lse && !aligned16(lse)))
    return set_error(DSA_ERR_INVALID_ARG, "dsa_csa_sparse_attn: pointers must be 16-byte aligned");
  dsa_status st = check_csa_shape("dsa_csa_sparse_attn", B, Lq, N_cmp, start_pos, m, k);
  if (st != DSA_OK) return st;
  if (n_h < 1 || D_qk < 1 || D_v < 1)
    return set_error(DSA_ERR_INVALID_ARG, "dsa_csa_sparse_attn: sizes must be positive");
  if (row_stride < D_qk || row_stride < D_v || row_stride % 8)
    return set_error(DSA_ERR_INVALID_ARG, "dsa_csa_sparse_attn: row stride must cover the row and be a multiple of 8");
  // Rows read min(t, k) index entries; the CSA rows hold at most
  // floor(t/m) valid entries below N_cmp and -1 after them.
  return sparse_attn_launch(q, c_cmp, row_stride, c_cmp, row_stride, idx, B, Lq, N_cmp, start_pos, n_h, D_qk, D_v,
                            k, scale, out, lse, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
