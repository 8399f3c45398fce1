// sparse_attn.cu -- sparse core attention over the selected positions.
//
// "注意力机制中的 Index" §2 (alpha-hat / o-hat: softmax over exactly S_t, then
// the weighted sum of the selected values) and §4 (MLA: every query head reads
// the same latent row c_s; K = the 576-wide latent row, V = its first 512
// columns).
//
// mla_sparse_attn_kernel (n_h = 128, D_qk = 576, D_v = 512, K = V = latent):
//   A cluster of two CTAs owns one query row (or one key-range split of it)
//   at a time.  CTA0 holds latent columns 0..255 of the query in TMEM, CTA1
//   columns 256..511 in TMEM and 512..575 in shared memory (the A operands of
//   the QK UMMAs); CTA c accumulates output columns 256c..256c+255 in TMEM
//   (fp32).  Per chunk of 64 selected rows:
//     6 producer warps  TMA gather4 of the chunk's latent rows (CTA0: 4 slabs
//                    of 64 columns, CTA1: 5 slabs) into the 128B-swizzled
//                    layout, 3-stage ring; each selected row is read from
//                    memory exactly once;
//     QK thread      S_c = Q_c K_c^T over the CTA's columns (A from TMEM) into
//                    a double-buffered S tile, as soon as the rows have
//                    landed and S two chunks back has been read;
//     PV thread      O_c += P V_c, P (bf16) from shared memory, V_c the
//                    gathered slabs 0..3 read as an MN-major B operand;
//     4 sender warps (thread = head) read S_c as soon as QK completes,
//                    stage it, fp32, in shared memory and ship each 16 KB
//                    half to the peer with one bulk copy as soon as it is
//                    staged (tx-counted on the peer's mbarrier of that half;
//                    the peer frees a half as soon as its softmax has read
//                    it); one of them loads the next row's query (TMA boxes
//                    through the staging tile, tcgen05.cp into TMEM) as soon
//                    as the last QK of the current row has completed;
//     8 softmax warps (thread = head = TMEM lane x half of the chunk) add the
//                    peer's partial (S = S_0 + S_1, identical in both CTAs as
//                    fp32 addition commutes), mask padded rows (fully valid
//                    chunks skip it), run the online softmax in the log2
//                    domain with lazy rescaling of O (only when the running
//                    max grows by more than 2^8), and write P as bf16 into a
//                    128B-swizzled K-major tile in shared memory.
//   The finished row is normalised by the softmax sum and stored as bf16.
//   Few long rows (decode) split the index list across clusters; the
//   partials (normalised O as bf16 pairs in a head-minor layout, so that the
//   thread-per-head epilogue stores whole 128-byte lines, and the log-sum-exp)
//   are combined by mla_merge_kernel, launched as a programmatic dependent of
//   the attention kernel so that its launch overlaps the attention tail.
//
// simt_sparse_attn_kernel: plain CUDA-core kernel for small head dims
// (D_qk, D_v <= 128, separate K and V tensors), one block per query row.
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>

#include "dsa_internal.h"
#include "dsa_ptx.cuh"

namespace dsa {

namespace {

// Sequence of a packed query row in a variable-length batch: the last b in
// [0, B) with cu_q[b] <= row (empty sequences share their successor's
// start, and the last of them owns the rows).
__device__ __forceinline__ int seq_of_row(const int* __restrict__ cu_q, int B, int row) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu_q + mid) <= row) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Where query row `row` sits: its sequence's first cached row, the cache
// length and the row's absolute position t.  Uniform batch (cu_q null): row
// = b * Lq + i at t = start_pos + i over rows b * Lk ...; varlen: from the
// prefix arrays.
struct RowPlace {
  int b, t, lk;
  long long kv_row0;
};
__device__ __forceinline__ RowPlace place_row(int row, int B, int Lq, int Lk, int start_pos, const int* cu_q,
                                              const int* cu_k, const int* sp) {
  RowPlace r;
  if (cu_q) {
    r.b = seq_of_row(cu_q, B, row);
    const int k0 = __ldg(cu_k + r.b);
    r.t = max(__ldg(sp + r.b), 0) + (row - __ldg(cu_q + r.b));
    r.lk = __ldg(cu_k + r.b + 1) - k0;
    r.kv_row0 = k0;
  } else {
    r.b = row / Lq;
    r.t = start_pos + row % Lq;
    r.lk = Lk;
    r.kv_row0 = static_cast<long long>(r.b) * Lk;
  }
  return r;
}

// ------------------------------------------------------------------ SIMT
constexpr int kSimtThreads = 128;

__global__ void __launch_bounds__(kSimtThreads)
simt_sparse_attn_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kb,
                        int64_t ks, const __nv_bfloat16* __restrict__ vb, int64_t vs,
                        const int32_t* __restrict__ idx, int B, int Lq, int Lk, int start_pos,
                        int n_h, int Dqk, int Dv, int k, float scale, __nv_bfloat16* __restrict__ out,
                        float* __restrict__ lse, const int* __restrict__ cu_q, const int* __restrict__ cu_k,
                        const int* __restrict__ sp) {
  extern __shared__ float qs[];  // [n_h][Dqk]
  pdl_trigger();
  pdl_wait();
  const size_t row = blockIdx.x;
  const RowPlace pl = place_row(static_cast<int>(row), B, Lq, Lk, start_pos, cu_q, cu_k, sp);
  const int nv = max(0, min(pl.t, k));
  for (int e = threadIdx.x; e < n_h * Dqk; e += kSimtThreads)
    qs[e] = __bfloat162float(q[row * n_h * Dqk + e]);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t* irow = idx + row * k;
  const __nv_bfloat16* kbase = kb + pl.kv_row0 * ks;
  const __nv_bfloat16* vbase = vb + pl.kv_row0 * vs;
  const float sl2 = scale * 1.4426950408889634f;
  for (int h = warp; h < n_h; h += kSimtThreads / 32) {
    float m = -INFINITY, l = 0.f;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int r = 0; r < nv; ++r) {
      const int s = irow[r];
      if (s < 0 || s >= pl.lk) continue;  // padding, or a position outside the sequence: skipped
      const __nv_bfloat16* kr = kbase + static_cast<int64_t>(s) * ks;
      float dot = 0.f;
      for (int c = lane; c < Dqk; c += 32) dot += qs[h * Dqk + c] * __bfloat162float(kr[c]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
      const float x = dot * sl2;
      const float mn = fmaxf(m, x);
      const float corr = exp2f(m - mn);
      const float p = exp2f(x - mn);
      l = l * corr + p;
      const __nv_bfloat16* vr = vbase + static_cast<int64_t>(s) * vs;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = lane + 32 * j;
        acc[j] = acc[j] * corr + (c < Dv ? p * __bfloat162float(vr[c]) : 0.f);
      }
      m = mn;
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = lane + 32 * j;
      if (c < Dv) out[(row * n_h + h) * Dv + c] = __float2bfloat16(acc[j] * inv);
    }
    if (lse && lane == 0) lse[row * n_h + h] = l > 0.f ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
  }
}

// ------------------------------------------------------------------ MLA
constexpr int kNH = 128, kDQK = 576, kDV = 512;
constexpr int kChunk = 64;                     // selected rows per chunk (UMMA N of QK)
constexpr int kSlabBytes = kChunk * 128;       // one 64-column slab of a chunk, 8 KB
constexpr int kMaxSlabs = 5;                   // CTA0: columns 0..255, CTA1: 256..575
constexpr int kStageBytes = kMaxSlabs * kSlabBytes;
constexpr int kStages = 3;
constexpr int kXBytes = kNH * kChunk * 4;      // partial score tile, fp32
constexpr int kXHalf = kXBytes / 2;            // one half: 32 columns of 128 heads, [head][32] fp32
constexpr int kPBytes = kNH * kChunk * 2;      // P tile, bf16, [head][64] 128B-swizzled (PV operand A)
constexpr int kQRopeBytes = kNH * 128;         // CTA1: query columns 512..575, bf16
constexpr int kQBoxBytes = kNH * 128;          // one TMA box of the query: 128 heads x 64 columns
// TMEM columns: O (fp32, 256) | S double buffer (fp32, 2 x 64) | Q (bf16 pairs, 128)
constexpr uint32_t kOCol = 0, kSCol = 256, kQCol = 384;
constexpr int kSoftWarps = 8;                  // warps 0..7
constexpr int kSendWarp0 = 8, kSendWarps = 4;  // warps 8..11
#ifndef MLA_PROD_WARPS
#define MLA_PROD_WARPS 6
#endif
constexpr int kProdWarp0 = 12, kProdWarps = MLA_PROD_WARPS;  // the chunk's 16 four-row groups
constexpr int kMmaWarpA = kProdWarp0 + kProdWarps;           // lane 0 issues QK
constexpr int kMmaWarpB = kMmaWarpA + 1;                     // lane 0 issues PV
constexpr int kMlaThreads = (kMmaWarpB + 1) * 32;            // 20 warps: 96 registers per thread
constexpr float kRescaleThresh = 8.0f;          // log2 units
constexpr int kPairBarBase = 2;                 // named barriers 2..5 and 6..9: the two softmax warps of a quadrant
constexpr int kSendBar = 10;                    // named barrier 10: the sender warps

struct MlaBars {
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], s_free[2];  // S tile computed / read by the softmax and sender warps
  uint64_t p_full, pv_done;       // P tile written / PV finished reading it (one phase per chunk)
  uint64_t o_full, o_free, q_full;
  uint64_t q_tma, q_cp;  // the item's query boxes landed / copied into TMEM (two phases per item)
  uint64_t x_full[2], x_free[2];  // per half of X_in: the peer's copy landed / the half consumed
  unsigned char kvmask[kStages][16];            // per 4-row group: validity bits
  float red[2][2][kNH];                         // [parity][half][head] chunk maxima
  float lsum[1][2][kNH];                        // [half][head] final sums
  uint32_t tmem_slot;
  int abort_flag;
};

// shared memory: gather ring | the peer's partials X_in (fp32) | this CTA's
// partials staged for the copies X_out | P | Q rope
constexpr int kMlaSmem = 1024 + kStages * kStageBytes + 2 * kXBytes + kPBytes + kQRopeBytes +
                         static_cast<int>(sizeof(MlaBars)) + 64;

struct MlaParams {
  const __nv_bfloat16* q;   // [B*Lq][128][576]
  const int32_t* idx;       // [B*Lq][k]
  __nv_bfloat16* out;       // [B*Lq][128][512]
  float* lse;               // [B*Lq][128] or null
  uint32_t* part_o;         // split partials, bf16 pairs: [B*Lq][S][256 column pairs][128 heads]
  float* part_lse;          // [B*Lq][S][128]
  unsigned int* err;
  const int* cu_q;          // variable-length batch (null: uniform)
  const int* cu_k;
  const int* sp;
  int B, Lq, Lk, start_pos, k;
  int rows;                 // query rows of the batch (B * Lq, or the packed total)
  int S, cps;               // key-range splits per row, chunks per split
  float scale_log2;
};

struct MlaItem {
  int row, split, c0, n;     // chunks [c0, c0 + n) of the row's index list
  int nv;                    // valid index entries read: min(t, k)
  int lk;                    // the sequence's cached rows
  int kv_row0;               // its first latent row in the tensor map
};

__device__ __forceinline__ MlaItem mla_item(const MlaParams& p, int item) {
  MlaItem it;
  it.row = item / p.S;
  it.split = item % p.S;
  const RowPlace pl = place_row(it.row, p.B, p.Lq, p.Lk, p.start_pos, p.cu_q, p.cu_k, p.sp);
  it.nv = max(0, min(pl.t, p.k));
  it.lk = pl.lk;
  it.kv_row0 = static_cast<int>(pl.kv_row0);
  const int nch = (it.nv + kChunk - 1) / kChunk;
  it.c0 = it.split * p.cps;
  it.n = max(0, min(nch, it.c0 + p.cps) - it.c0);
  return it;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kMlaThreads, 1)
mla_sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_kv, const __grid_constant__ CUtensorMap tm_q,
                       const MlaParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* kv_smem = smem;
  uint8_t* xin_smem = kv_smem + kStages * kStageBytes;   // X_in[half]: the peer's partials
  uint8_t* xout_smem = xin_smem + kXBytes;               // X_out[half]: this CTA's, staged
  uint8_t* p_smem = xout_smem + kXBytes;                 // P of the current chunk
  uint8_t* qrope_smem = p_smem + kPBytes;                // CTA1: Q[:, 512:576]
  MlaBars* bb = reinterpret_cast<MlaBars*>(qrope_smem + kQRopeBytes);
  volatile int* abort_flag = &bb->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;
  const int n_items = p.rows * p.S;
  // CTA0 owns latent columns 0..255 (QK and V), CTA1 owns 256..575 (QK) and
  // 256..511 (V); together they gather each selected row exactly once.
  const int n_slabs = rank == 0 ? 4 : 5;
  const int col0 = rank == 0 ? 0 : 256;

  if (threadIdx.x == 0) {
    // kv_full: one arrive.expect_tx per 4-row group issuer
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bb->kv_full[s], kChunk / 4);
      mbar_init(&bb->kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bb->s_full[b], 1);
      mbar_init(&bb->s_free[b], kSoftWarps + kSendWarps);
      // X_in half b: the peer's bulk copy completes the phase; the phase of
      // chunk 0 is armed here, the next one by the softmax warps of that half
      // as they consume a chunk
      mbar_init(&bb->x_full[b], 1);
      mbar_init(&bb->x_free[b], kSoftWarps / 2);
      mbar_arrive_expect_tx(&bb->x_full[b], kXHalf);
    }
    mbar_init(&bb->p_full, kSoftWarps);
    mbar_init(&bb->pv_done, 1);
    mbar_init(&bb->o_full, 1);
    mbar_init(&bb->o_free, kSoftWarps);
    mbar_init(&bb->q_full, 1);
    mbar_init(&bb->q_tma, 1);
    mbar_init(&bb->q_cp, 1);
    bb->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarpA) {
    tmem_alloc(&bb->tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = bb->tmem_slot;
  // the next kernel may be scheduled now (it waits for this grid before
  // touching memory); this grid waits for the previous one likewise
  pdl_trigger();
  pdl_wait();

  if (warp >= kProdWarp0 && warp < kProdWarp0 + kProdWarps) {
    // ------------------------------------------------------------ gather
    // TMA gather4 of the chunk's selected latent rows into the 128B-swizzled
    // slab layout the UMMAs read.  Gather throughput grows with the number of
    // issuing warps, so kProdWarps warps share each chunk's 16 four-row groups:
    // warp pw owns groups pw + kProdWarps * i (i = 0, 1, 2, when < 16); lane i
    // issues group pw + kProdWarps * i over all slabs after lanes 4i..4i+3
    // fetched its row indices.
    const int pw = warp - kProdWarp0;
    const int n_groups = pw + 2 * kProdWarps < 16 ? 3 : 2;
    uint32_t g = 0;  // global chunk counter
    bool ok = true;
    for (int item = pair; item < n_items && ok; item += n_pairs) {
      const MlaItem it = mla_item(p, item);
      if (it.n == 0) continue;
      const int32_t* irow = p.idx + static_cast<size_t>(it.row) * p.k;
      const int row_base = it.kv_row0;
      const int my_group = pw + kProdWarps * (lane >> 2);   // group whose row this lane fetches
      auto fetch = [&](int c) -> int {
        const int r = c * kChunk + my_group * 4 + (lane & 3);
        return ((lane >> 2) < n_groups && r < it.nv) ? __ldg(irow + r) : -1;
      };
      // indices are fetched three chunks ahead (decode items are a few chunks
      // long, so their whole index list is in flight at once)
      const int c_end = it.c0 + it.n;
      int f0 = fetch(it.c0);
      int f1 = it.c0 + 1 < c_end ? fetch(it.c0 + 1) : -1;
      int f2 = it.c0 + 2 < c_end ? fetch(it.c0 + 2) : -1;
      for (int c = it.c0; c < c_end; ++c, ++g) {
        const int stage = g % kStages;
        const uint32_t ph = (g / kStages) & 1;
        const int sidx = f0;
        f0 = f1;
        f1 = f2;
        f2 = c + 3 < c_end ? fetch(c + 3) : -1;
        const bool valid = sidx >= 0 && sidx < it.lk;
        const int grow = row_base + (valid ? sidx : 0);   // padded rows read row 0 (masked later)
        const unsigned m = __ballot_sync(0xffffffffu, valid);
        const int src = (lane < n_groups ? lane : 0) * 4;
        const int r0 = __shfl_sync(0xffffffffu, grow, src + 0);
        const int r1 = __shfl_sync(0xffffffffu, grow, src + 1);
        const int r2 = __shfl_sync(0xffffffffu, grow, src + 2);
        const int r3 = __shfl_sync(0xffffffffu, grow, src + 3);
        const bool w = __all_sync(0xffffffffu, mbar_wait(&bb->kv_empty[stage], ph ^ 1, abort_flag));
        if (!w) { ok = false; break; }  // warp-uniform
        if (lane < n_groups) {
          const int grp = pw + kProdWarps * lane;
          bb->kvmask[stage][grp] = static_cast<unsigned char>((m >> (4 * lane)) & 0xFu);
          uint8_t* dst = kv_smem + stage * kStageBytes + grp * 512;
          mbar_arrive_expect_tx(&bb->kv_full[stage], n_slabs * 512);
          for (int sl = 0; sl < n_slabs; ++sl)
            tma_gather4(dst + sl * kSlabBytes, &tm_kv, &bb->kv_full[stage], col0 + sl * 64, r0, r1, r2, r3);
        }
      }
    }
  } else if (warp == kMmaWarpA) {
    // ------------------------------------------------------------ MMA: QK
    // S[g & 1] = Q K(g)^T as soon as the chunk's rows have landed and the
    // softmax and sender warps have read S(g - 2) out of that buffer.
    if (lane == 0) {
      uint32_t g = 0, it_n = 0;
      bool ok = true;
      const uint32_t idesc_qk = make_idesc_bf16(128, kChunk, 0, 0);
      const uint32_t qrope_base = smem_u32(qrope_smem);
      for (int item = pair; item < n_items && ok; item += n_pairs) {
        const MlaItem it = mla_item(p, item);
        if (it.n == 0) continue;
        if (!mbar_wait(&bb->q_full, it_n & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int c = 0; c < it.n; ++c, ++g) {
          const int stage = g % kStages;
          if (!mbar_wait(&bb->kv_full[stage], (g / kStages) & 1, abort_flag) ||
              !mbar_wait(&bb->s_free[g & 1], ((g >> 1) & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t kb = smem_u32(kv_smem + stage * kStageBytes);
          const uint32_t s_col = kSCol + (g & 1) * 64;
#pragma unroll
          for (int st = 0; st < 16; ++st) {
            const uint64_t bd = make_smem_desc(kb + (st >> 2) * kSlabBytes + (st & 3) * 32, 16, 1024,
                                               kSwizzle128B);
            umma_bf16_ts(tmem + s_col, tmem + kQCol + st * 8, bd, idesc_qk, st != 0);
          }
          if (rank == 1) {
            // query columns 512..575 from shared memory against slab 4
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = make_smem_desc(qrope_base + kk * 32, 16, 1024, kSwizzle128B);
              const uint64_t bd = make_smem_desc(kb + 4 * kSlabBytes + kk * 32, 16, 1024, kSwizzle128B);
              umma_bf16_ss(tmem + s_col, ad, bd, idesc_qk, 1u);
            }
          }
          umma_commit(&bb->s_full[g & 1]);
        }
        ++it_n;
      }
    }
  } else if (warp == kMmaWarpB) {
    // ------------------------------------------------------------ MMA: PV
    // O += P(g) V(g), P (bf16) from shared memory, V = this CTA's slabs 0..3:
    // value columns 0..255 (CTA0) or 256..511 (CTA1).
    if (lane == 0) {
      uint32_t g = 0, it_n = 0;
      bool ok = true;
      const uint32_t idesc_pv = make_idesc_bf16(128, 256, 0, 1);
      const uint32_t p_base = smem_u32(p_smem);
      for (int item = pair; item < n_items && ok; item += n_pairs) {
        const MlaItem it = mla_item(p, item);
        if (it.n == 0) continue;
        for (int c = 0; c < it.n; ++c, ++g) {
          const int stage = g % kStages;
          if (!mbar_wait(&bb->p_full, g & 1, abort_flag) ||
              (c == 0 && !mbar_wait(&bb->o_free, (it_n & 1) ^ 1, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t v_base = smem_u32(kv_smem + stage * kStageBytes);
#pragma unroll
          for (int kk = 0; kk < kChunk / 16; ++kk) {
            const uint64_t ad = make_smem_desc(p_base + kk * 32, 16, 1024, kSwizzle128B);
            const uint64_t bd = make_smem_desc(v_base + kk * 2048, kSlabBytes, 1024, kSwizzle128B);
            umma_bf16_ss(tmem + kOCol, ad, bd, idesc_pv, (c == 0 && kk == 0) ? 0u : 1u);
          }
          umma_commit(&bb->pv_done);
          umma_commit(&bb->kv_empty[stage]);
        }
        if (!ok) break;
        umma_commit(&bb->o_full);
        ++it_n;
      }
    }
  } else if (warp >= kSendWarp0) {
    // ------------------------------------------------------------ sender
    // thread = head (TMEM lane); loads the CTA's query part at item start and
    // ships every chunk's partial scores to the peer as soon as QK finishes,
    // so the exchange overlaps the softmax of the previous chunk.
    const int qd = warp - kSendWarp0;
    const int h = qd * 32 + lane;
    const int stid = threadIdx.x - kSendWarp0 * 32;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    const uint32_t xin_remote = mapa_shared(smem_u32(xin_smem), peer);
    uint32_t q_phase = 0;  // completed phases of q_tma and q_cp
    const uint32_t xfull_remote0 = mapa_shared(smem_u32(&bb->x_full[0]), peer);
    const uint32_t xfull_remote1 = mapa_shared(smem_u32(&bb->x_full[1]), peer);
    // A failed (timed-out) wait only clears `ok`; the sender warps leave their
    // loops together, at the next named barrier, so none is left waiting there.
    uint32_t g = 0, it_n = 0;
    bool ok = true;
    for (int item = pair; item < n_items; item += n_pairs) {
      const MlaItem it = mla_item(p, item);
      if (it.n == 0) continue;
      // Q's TMEM columns (and CTA1's rope tile) are free: this warp saw the
      // previous item's last S, so every QK of that item has completed (no
      // later MMA of it reads Q).  One thread brings the CTA's query part in:
      // TMA boxes of 128 heads x 64 columns (128B-swizzled, two at a time
      // through the idle staging buffer X_out) and tcgen05.cp into TMEM, in
      // the layout the QK MMA reads; CTA1's rope columns land directly in
      // their shared-memory tile.  The load overlaps the item's last softmax,
      // PV and epilogue.
      tc_fence_after();
      if (stid == 0 && ok) {
        bulk_wait_read_all();  // the previous chunk's copies have read X_out
        const int qrow = it.row * kNH;
#pragma unroll 1
        for (int pass = 0; pass < 2 && ok; ++pass) {
          const uint32_t bytes = 2 * kQBoxBytes + (rank == 1 && pass == 0 ? kQRopeBytes : 0);
          mbar_arrive_expect_tx(&bb->q_tma, bytes);
          for (int b = 0; b < 2; ++b)
            tma_load_2d(xout_smem + b * kQBoxBytes, &tm_q, &bb->q_tma, col0 + (2 * pass + b) * 64, qrow);
          if (rank == 1 && pass == 0) tma_load_2d(qrope_smem, &tm_q, &bb->q_tma, 512, qrow);
          ok = mbar_wait(&bb->q_tma, q_phase & 1, abort_flag);
          if (ok) {
            tc_fence_after();
            for (int b = 0; b < 2; ++b)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                tc_cp_128x256b(tmem + kQCol + (2 * pass + b) * 32 + kk * 8,
                               make_smem_desc(smem_u32(xout_smem + b * kQBoxBytes) + kk * 32, 16, 1024,
                                              kSwizzle128B));
            umma_commit(&bb->q_cp);
            ok = mbar_wait(&bb->q_cp, q_phase & 1, abort_flag);  // X_out read, TMEM written
          }
          ++q_phase;
        }
        tc_fence_before();
        if (ok) mbar_arrive(&bb->q_full);
      }
      __syncwarp();
      // this head's part of the next item's query, warmed into L2 a few chunks
      // before it is loaded (earlier, the gathers would evict it again)
      const char* nq = item + n_pairs < n_items
                           ? reinterpret_cast<const char*>(
                                 p.q + (static_cast<size_t>((item + n_pairs) / p.S) * kNH + h) * kDQK + col0)
                           : nullptr;
      const int c_pf = max(0, it.n - 8);
      for (int c = 0; c < it.n; ++c, ++g) {
        const int sb = g & 1;
        if (c == c_pf && nq != nullptr)
          for (int ln = 0; ln < (rank == 0 ? 4 : 5); ++ln) prefetch_l2(nq + ln * 128);
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bb->s_full[sb], (g >> 1) & 1, abort_flag));
        tc_fence_after();
        // X_out is free once the previous chunk's copies have read it
        if (stid == 0) bulk_wait_read_all();
        ok = named_bar_and(kSendBar, kSendWarps * 32, ok);
        if (ok) {
          // row h of each 32-column half: 16-byte pieces XOR-swizzled by
          // h & 7, so that the peer's per-head reads are free of bank conflicts
#pragma unroll 1
          for (int half = 0; half < 2; ++half) {
            uint32_t v[32];
            tmem_ld32<32>(t_lane + kSCol + sb * 64 + half * 32, v);
            tmem_ld_wait();
            uint8_t* xo = xout_smem + half * kXHalf + h * 128;
#pragma unroll
            for (int j = 0; j < 8; ++j)
              *reinterpret_cast<uint4*>(xo + ((j ^ (h & 7)) << 4)) =
                  make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          }
        }
        // S(g) has been read: QK(g + 2) may overwrite the buffer
        tc_fence_before();
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(&bb->s_free[sb]);
        fence_proxy_async_smem();
        named_bar_sync(kSendBar + 1, kSendWarps * 32);
        if (stid == 0 && ok) {
          // each half of the peer's X_in is free once the peer's softmax warps
          // of that half have consumed chunk g - 1
#pragma unroll 1
          for (int half = 0; half < 2 && ok; ++half) {
            if (mbar_wait_cluster(&bb->x_free[half], (g & 1) ^ 1, abort_flag)) {
              bulk_copy_to_peer(xin_remote + half * kXHalf, smem_u32(xout_smem) + half * kXHalf, kXHalf,
                                half ? xfull_remote1 : xfull_remote0);
              bulk_commit_group();
            } else {
              ok = false;  // the abort flag is raised; the next barrier ends the loop
            }
          }
        }
      }
      ok = named_bar_and(kSendBar, kSendWarps * 32, ok);
      if (!ok) break;
      ++it_n;
    }
    if (stid == 0) bulk_wait_read_all();  // the last copies have read the staging buffer
  } else {
    // ------------------------------------------------------------ softmax
    // thread = (head h = TMEM lane, half hf of the chunk's 64 columns)
    const int qd = warp & 3, hf = warp >> 2;
    const int h = qd * 32 + lane;
    const int pair_bar = kPairBarBase + qd;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    const uint32_t xfree_remote = mapa_shared(smem_u32(&bb->x_free[hf]), peer);
    // A failed (timed-out) wait only clears `ok`; the two warps of a head pair
    // leave their loops together at the next pair barrier.
    uint32_t g = 0, it_n = 0;
    bool ok = true;
    for (int item = pair; item < n_items; item += n_pairs) {
      const MlaItem it = mla_item(p, item);
      const bool partial = p.S > 1;
      if (it.n == 0) {
        if (partial) {
          uint32_t* po = p.part_o + ((static_cast<size_t>(it.row) * p.S + it.split) * 256 + rank * 128 + hf * 64) * kNH + h;
          for (int j = 0; j < 64; ++j) po[j * kNH] = 0u;
          if (rank == 0 && hf == 0)
            p.part_lse[(static_cast<size_t>(it.row) * p.S + it.split) * kNH + h] = -INFINITY;
        } else {
          __nv_bfloat16* orow = p.out + (static_cast<size_t>(it.row) * kNH + h) * kDV + rank * 256 + hf * 128;
          for (int j = 0; j < 16; ++j) reinterpret_cast<uint4*>(orow)[j] = make_uint4(0, 0, 0, 0);
          if (p.lse && rank == 0 && hf == 0) p.lse[static_cast<size_t>(it.row) * kNH + h] = -INFINITY;
        }
        continue;
      }
      // l_run: softmax denominator (fp32, before the bf16 rounding of P); each
      // half of a head keeps the sum of its own columns.
      float m_run = -INFINITY, l_run = 0.f;
      for (int c = 0; c < it.n; ++c, ++g) {
        const int stage = g % kStages;
        const int sb = g & 1;
        float s[32];
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bb->s_full[sb], (g >> 1) & 1, abort_flag));
        tc_fence_after();
        if (ok) {
          uint32_t v[32];
          tmem_ld32<32>(t_lane + kSCol + sb * 64 + hf * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) s[j] = __uint_as_float(v[j]);
        }
        // S(g) has been read: QK(g + 2) may overwrite the buffer
        tc_fence_before();
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(&bb->s_free[sb]);
        // the rows' validity bits (eight 4-bit group masks, one per byte ->
        // 32 row bits), read while the peer's partials are in flight
        if (ok) ok = mbar_wait(&bb->kv_full[stage], (g / kStages) & 1, abort_flag);
        uint32_t vm = 0xFFFFFFFFu;
        if (ok) {
          uint64_t x = *reinterpret_cast<const uint64_t*>(&bb->kvmask[stage][8 * hf]) & 0x0F0F0F0F0F0F0F0Full;
          x = (x | (x >> 4)) & 0x00FF00FF00FF00FFull;
          x = (x | (x >> 8)) & 0x0000FFFF0000FFFFull;
          x = (x | (x >> 16)) & 0x00000000FFFFFFFFull;
          vm = static_cast<uint32_t>(x);
        }
        // + the peer's partial scores of the same columns (fp32)
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait_cluster(&bb->x_full[hf], g & 1, abort_flag));
        if (ok) {
          const uint8_t* xr = xin_smem + hf * kXHalf + h * 128;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 o = *reinterpret_cast<const float4*>(xr + ((j ^ (h & 7)) << 4));
            s[4 * j] += o.x;
            s[4 * j + 1] += o.y;
            s[4 * j + 2] += o.z;
            s[4 * j + 3] += o.w;
            // the raw maximum of a fully valid chunk, in four chains while
            // the loads are in flight
            m4[0] = fmaxf(m4[0], s[4 * j]);
            m4[1] = fmaxf(m4[1], s[4 * j + 1]);
            m4[2] = fmaxf(m4[2], s[4 * j + 2]);
            m4[3] = fmaxf(m4[3], s[4 * j + 3]);
          }
        }
        // this half of X_in is consumed (the additions above used every loaded
        // value): arm its phase for the next chunk, then let the peer send it
        __syncwarp();
        if (qd == 0 && lane == 0 && ok) mbar_arrive_expect_tx(&bb->x_full[hf], kXHalf);
        if (lane == 0 && ok) mbar_arrive_remote_relaxed(xfree_remote);
        // mask, scale, chunk max (combined with the other half of the head);
        // the scale (> 0) is applied to the maximum and inside the exponent
        // with one FMA per element
        float lmax = -INFINITY;
        if (ok) {
          if (vm != 0xFFFFFFFFu) {  // warp-uniform: rows are the same for every head
#pragma unroll
            for (int j = 0; j < 32; ++j) s[j] = ((vm >> j) & 1u) ? s[j] : -INFINITY;
            // max of the masked scores as a tree (short dependency chains)
            float m8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) m8[j] = fmaxf(fmaxf(s[j], s[j + 8]), fmaxf(s[j + 16], s[j + 24]));
            lmax = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
          } else {
            lmax = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
          }
        }
        bb->red[g & 1][hf][h] = lmax;
        // PV(g - 1) has read P(g - 1) (and O holds it): checked while the
        // other half of the head reaches the pair barrier, before P(g) and
        // any rescale of O
        if (ok && g > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bb->pv_done, (g - 1) & 1, abort_flag));
        ok = named_bar_and(pair_bar, 64, ok);
        if (!ok) break;
        const float cmax = fmaxf(lmax, bb->red[g & 1][hf ^ 1][h]) * p.scale_log2;
        // Heads rescale independently, but the TMEM accesses below are
        // warp-collective (.sync.aligned): the warp enters together when any
        // of its heads needs it, and the others scale by exactly 1.
        const bool grow = cmax > m_run + kRescaleThresh;
        if (__any_sync(0xffffffffu, grow)) {
          const float factor = grow ? ex2_approx(m_run - cmax) : 1.f;  // 0 when m_run = -inf
          if (c > 0) {
            // O holds PV of the earlier chunks (PV(g - 1) has completed: see
            // above): scale my 128 columns
            tc_fence_after();
            if (ok) {
#pragma unroll 1
              for (int blk = 0; blk < 4; ++blk) {
                uint32_t v[32];
                const uint32_t col = kOCol + hf * 128 + blk * 32;
                tmem_ld32<32>(t_lane + col, v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * factor);
                tmem_st32x32(t_lane + col, v);
              }
              tmem_st_wait();
            }
          }
          if (grow) {
            l_run *= factor;
            m_run = cmax;
          }
        }
        uint32_t pk[16];
        float e4[4] = {0.f, 0.f, 0.f, 0.f};  // four partial sums (short chains)
        const bool live = m_run != -INFINITY;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float a = live ? ex2_approx(fmaf(s[2 * j], p.scale_log2, -m_run)) : 0.f;
          const float bq = live ? ex2_approx(fmaf(s[2 * j + 1], p.scale_log2, -m_run)) : 0.f;
          const __nv_bfloat162 pr = __floats2bfloat162_rn(a, bq);
          e4[j & 3] += a + bq;
          pk[j] = *reinterpret_cast<const uint32_t*>(&pr);
        }
        l_run += (e4[0] + e4[1]) + (e4[2] + e4[3]);
        // P(g) overwrites P(g - 1), which PV(g - 1) has read (checked above):
        // row h of the 128B-swizzled K-major tile, this half's 64 bytes as
        // four 16-byte pieces
        if (ok) {
          uint8_t* prow = p_smem + h * 128;
#pragma unroll
          for (int i = 0; i < 4; ++i)
            *reinterpret_cast<uint4*>(prow + (((hf * 4 + i) ^ (h & 7)) << 4)) =
                make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          fence_proxy_async_smem();
        }
        tc_fence_before();  // orders a rescale's TMEM stores before PV(g)
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(&bb->p_full);
      }
      // combine the two halves' sums
      bb->lsum[0][hf][h] = l_run;
      ok = named_bar_and(pair_bar, 64, ok);
      if (!ok) break;
      const float l_tot = l_run + bb->lsum[0][hf ^ 1][h];
      const float l_lse_tot = l_tot;
      named_bar_sync(pair_bar + 4, 64);  // lsum is rewritten by the next item
      // epilogue: O / l
      ok = __all_sync(0xffffffffu, mbar_wait(&bb->o_full, it_n & 1, abort_flag));
      tc_fence_after();
      const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
      const float lse_v = l_lse_tot > 0.f ? (m_run + __log2f(l_lse_tot)) * 0.6931471805599453f : -INFINITY;
      if (ok && !partial) {
        __nv_bfloat16* orow = p.out + (static_cast<size_t>(it.row) * kNH + h) * kDV + rank * 256 + hf * 128;
#pragma unroll 1
        for (int blk = 0; blk < 4; ++blk) {
          uint32_t v[32];
          tmem_ld32<32>(t_lane + kOCol + hf * 128 + blk * 32, v);
          tmem_ld_wait();
          uint32_t o[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const __nv_bfloat162 pr = __floats2bfloat162_rn(__uint_as_float(v[2 * j]) * inv,
                                                            __uint_as_float(v[2 * j + 1]) * inv);
            o[j] = *reinterpret_cast<const uint32_t*>(&pr);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow + blk * 32);
#pragma unroll
          for (int j = 0; j < 4; ++j) dst[j] = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
        }
        if (p.lse && rank == 0 && hf == 0) p.lse[static_cast<size_t>(it.row) * kNH + h] = lse_v;
      } else if (ok) {
        const size_t slot = static_cast<size_t>(it.row) * p.S + it.split;
        // column pair cp of head h at word (cp, h): a warp stores 128 contiguous bytes
        uint32_t* po = p.part_o + (slot * 256 + rank * 128 + hf * 64) * kNH + h;
#pragma unroll 1
        for (int blk = 0; blk < 4; ++blk) {
          uint32_t v[32];
          tmem_ld32<32>(t_lane + kOCol + hf * 128 + blk * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const __nv_bfloat162 pr = __floats2bfloat162_rn(__uint_as_float(v[2 * j]) * inv,
                                                            __uint_as_float(v[2 * j + 1]) * inv);
            po[(blk * 16 + j) * kNH] = *reinterpret_cast<const uint32_t*>(&pr);
          }
        }
        if (rank == 0 && hf == 0) p.part_lse[slot * kNH + h] = lse_v;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive(&bb->o_free);
      ++it_n;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) atomicOr(p.err, 1u);
  // neither CTA may leave while its peer can still touch its shared memory
  cluster_sync();
  if (warp == kMmaWarpA) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Combines the S key-range partials of each row: out = sum_j w_j o_j with
// w_j = exp(lse_j - LSE), LSE = log sum_j exp(lse_j).  Block (row, cb) makes
// output columns 16 cb .. 16 cb + 15 of all 128 heads: partial words are read
// along the head (contiguous), the result is transposed in shared memory and
// stored as 32-byte pieces of the head rows.
constexpr int kMergeThreads = 256;
constexpr int kMergeCols = 16;
constexpr int kMaxMergeSplits = 32;
__global__ void __launch_bounds__(kMergeThreads)
mla_merge_kernel(const uint32_t* __restrict__ part_o, const float* __restrict__ part_lse,
                 __nv_bfloat16* __restrict__ out, float* __restrict__ lse, int S) {
  // the partials are written by the attention grid this launch depends on
  pdl_trigger();
  pdl_wait();
  const size_t row = blockIdx.x;
  const int cb = blockIdx.y;
  __shared__ float wgt[kMaxMergeSplits][kNH];
  __shared__ uint32_t tile[kNH][kMergeCols / 2 + 1];
  const int t = threadIdx.x;
  constexpr int kPairs = kMergeCols / 4;  // column pairs per thread (two threads per head)
  const int h = t & (kNH - 1), half = t >> 7;
  const int cp0 = cb * (kMergeCols / 2) + half * kPairs;
  // the first kPre splits' partial words are loaded before the weights are
  // known, so that both global round trips overlap
  constexpr int kPre = 8;
  uint32_t pre[kPre][kPairs];
#pragma unroll
  for (int j = 0; j < kPre; ++j) {
    if (j < S) {
      const uint32_t* src = part_o + ((row * S + j) * 256 + cp0) * kNH + h;
#pragma unroll
      for (int i = 0; i < kPairs; ++i) pre[j][i] = src[i * kNH];
    }
  }
  for (int e = t; e < S * kNH; e += kMergeThreads) wgt[e / kNH][e % kNH] = part_lse[row * S * kNH + e];
  __syncthreads();
  if (t < kNH) {
    float m = -INFINITY;
    for (int j = 0; j < S; ++j) m = fmaxf(m, wgt[j][t]);
    float z = 0.f;
    for (int j = 0; j < S; ++j) {
      const float e = m == -INFINITY ? 0.f : __expf(wgt[j][t] - m);
      wgt[j][t] = e;
      z += e;
    }
    const float iz = z > 0.f ? 1.f / z : 0.f;
    for (int j = 0; j < S; ++j) wgt[j][t] *= iz;
    if (lse && cb == 0) lse[row * kNH + t] = z > 0.f ? m + __logf(z) : -INFINITY;
  }
  __syncthreads();
  float acc[2 * kPairs];
#pragma unroll
  for (int i = 0; i < 2 * kPairs; ++i) acc[i] = 0.f;
#pragma unroll
  for (int j = 0; j < kPre; ++j) {
    if (j < S) {
      const float wj = wgt[j][h];
#pragma unroll
      for (int i = 0; i < kPairs; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pre[j][i]));
        acc[2 * i] = fmaf(wj, f.x, acc[2 * i]);
        acc[2 * i + 1] = fmaf(wj, f.y, acc[2 * i + 1]);
      }
    }
  }
#pragma unroll 4
  for (int j = kPre; j < S; ++j) {
    const float wj = wgt[j][h];
    const uint32_t* src = part_o + ((row * S + j) * 256 + cp0) * kNH + h;
    uint32_t wv[kPairs];
#pragma unroll
    for (int i = 0; i < kPairs; ++i) wv[i] = src[i * kNH];
#pragma unroll
    for (int i = 0; i < kPairs; ++i) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[i]));
      acc[2 * i] = fmaf(wj, f.x, acc[2 * i]);
      acc[2 * i + 1] = fmaf(wj, f.y, acc[2 * i + 1]);
    }
  }
#pragma unroll
  for (int i = 0; i < kPairs; ++i) {
    const __nv_bfloat162 pr = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    tile[h][half * kPairs + i] = *reinterpret_cast<const uint32_t*>(&pr);
  }
  __syncthreads();
  uint32_t* orow = reinterpret_cast<uint32_t*>(out + row * kNH * kDV) + cb * (kMergeCols / 2);
  for (int e = t; e < kNH * (kMergeCols / 2); e += kMergeThreads) {
    const int hh = e / (kMergeCols / 2), w = e % (kMergeCols / 2);
    orow[hh * (kDV / 2) + w] = tile[hh][w];
  }
}

struct MlaSplit {
  int S, cps, pairs;
};

MlaSplit mla_split(long long rows, int k, int sms) {
  MlaSplit sp{};
  const int max_pairs = std::max(1, sms / 2);
  const int nch = std::max(1, (k + kChunk - 1) / kChunk);
  sp.S = 1;
  sp.cps = nch;
  if (rows < max_pairs) {
    int S = static_cast<int>(std::min<long long>(32, max_pairs / rows));
    S = std::max(1, std::min(S, nch));
    sp.cps = (nch + S - 1) / S;
    sp.S = (nch + sp.cps - 1) / sp.cps;
  }
  sp.pairs = static_cast<int>(std::min<long long>(rows * sp.S, max_pairs));
  return sp;
}

}  // namespace

size_t sparse_attn_ws_rows(long long rows, int n_h, int D_v, int k) {
  if (n_h != kNH || D_v != kDV) return 0;
  // sized for up to 160 SMs so the requirement does not depend on the device
  const MlaSplit sp = mla_split(rows, k, 160);
  if (sp.S <= 1) return 0;
  return static_cast<size_t>(rows) * sp.S * kNH * (kDV / 2 + 1) * 4 + 256;
}

size_t sparse_attn_ws_bytes(int B, int Lq, int n_h, int D_v, int k) {
  return sparse_attn_ws_rows(static_cast<long long>(B) * Lq, n_h, D_v, k);
}

dsa_status sparse_attn_launch(const dsa_bf16* q, const dsa_bf16* kbuf, int64_t k_row_stride,
                              const dsa_bf16* vbuf, int64_t v_row_stride, const int32_t* idx,
                              int B, int Lq, int Lk, int start_pos, int n_h, int D_qk, int D_v,
                              int k, float scale, dsa_bf16* out, float* lse, void* ws,
                              size_t ws_bytes, cudaStream_t stream, const VarlenArgs* vl) {
  const long long rows = vl ? static_cast<long long>(vl->total_q) : static_cast<long long>(B) * Lq;
  const long long kv_rows = vl ? static_cast<long long>(vl->total_k) : static_cast<long long>(B) * Lk;
  if (rows > (1ll << 31) - 1) return set_error(DSA_ERR_UNSUPPORTED, "dsa_sparse_attn: too many rows");
  const bool mla = n_h == kNH && D_qk == kDQK && D_v == kDV && kbuf == vbuf &&
                   k_row_stride == v_row_stride;
  if (mla) {
    const int sms = device_sm_count();
    if (sms <= 0) return set_error(DSA_ERR_CUDA, "cannot query the device SM count");
    const MlaSplit sp = mla_split(rows, k, std::min(sms, 160));
    if (rows * sp.S > (1ll << 31) - 1) return set_error(DSA_ERR_UNSUPPORTED, "dsa_sparse_attn: too many rows");
    const size_t need = sp.S > 1 ? static_cast<size_t>(rows) * sp.S * kNH * (kDV / 2 + 1) * 4 : 0;
    if (need > ws_bytes || (need && !ws)) return set_error(DSA_ERR_WORKSPACE, "dsa_sparse_attn: workspace too small");
    CUtensorMap tkv, tq;
    if (!encode_tiled_2d(&tkv, kbuf, kDQK, static_cast<uint64_t>(kv_rows),
                         static_cast<uint64_t>(k_row_stride) * 2, 64, 1, CU_TENSOR_MAP_SWIZZLE_128B))
      return set_error(DSA_ERR_CUDA, "tensor map for the latent cache failed");
    // the query as [rows * 128 heads][576] with boxes of 128 heads x 64 columns
    if (!encode_tiled_2d(&tq, q, kDQK, static_cast<uint64_t>(rows) * kNH, kDQK * 2, 64, kNH,
                         CU_TENSOR_MAP_SWIZZLE_128B))
      return set_error(DSA_ERR_CUDA, "tensor map for the query failed");
    MlaParams p{};
    p.q = reinterpret_cast<const __nv_bfloat16*>(q);
    p.idx = idx;
    p.out = reinterpret_cast<__nv_bfloat16*>(out);
    p.lse = lse;
    p.part_o = sp.S > 1 ? static_cast<uint32_t*>(ws) : nullptr;
    p.part_lse = sp.S > 1 ? reinterpret_cast<float*>(static_cast<uint32_t*>(ws) +
                                                     static_cast<size_t>(rows) * sp.S * kNH * (kDV / 2))
                          : nullptr;
    p.err = device_error_word();
    if (!p.err) return set_error(DSA_ERR_CUDA, "cannot resolve the device error word");
    p.cu_q = vl ? vl->cu_q : nullptr;
    p.cu_k = vl ? vl->cu_k : nullptr;
    p.sp = vl ? vl->sp : nullptr;
    p.B = B; p.Lq = Lq; p.Lk = Lk; p.start_pos = start_pos; p.k = k;
    p.rows = static_cast<int>(rows);
    p.S = sp.S; p.cps = sp.cps;
    p.scale_log2 = scale * 1.4426950408889634f;
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(mla_sparse_attn_kernel), kMlaSmem);
    if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("mla smem attribute: ") + cudaGetErrorString(e));
    e = launch_pdl(mla_sparse_attn_kernel, dim3(static_cast<unsigned>(2 * sp.pairs)), dim3(kMlaThreads), kMlaSmem,
                   stream, tkv, tq, p);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("mla launch: ") + cudaGetErrorString(e));
    if (sp.S > 1) {
      e = launch_pdl(mla_merge_kernel, dim3(static_cast<unsigned>(rows), kDV / kMergeCols), dim3(kMergeThreads), 0,
                     stream, static_cast<const uint32_t*>(p.part_o), static_cast<const float*>(p.part_lse), p.out,
                     lse, sp.S);
      if (e == cudaSuccess) e = cudaGetLastError();
      if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("mla merge launch: ") + cudaGetErrorString(e));
    }
    return DSA_OK;
  }
  if (n_h <= 128 && D_qk <= 128 && D_v <= 128) {
    const int smem = n_h * D_qk * 4;
    if (smem > 48 * 1024) {
      cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(simt_sparse_attn_kernel), smem);
      if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("simt smem attribute: ") + cudaGetErrorString(e));
    }
    cudaError_t e = launch_pdl(simt_sparse_attn_kernel, dim3(static_cast<unsigned>(rows)), dim3(kSimtThreads), smem,
                               stream, reinterpret_cast<const __nv_bfloat16*>(q),
                               reinterpret_cast<const __nv_bfloat16*>(kbuf), k_row_stride,
                               reinterpret_cast<const __nv_bfloat16*>(vbuf), v_row_stride, idx, B, Lq, Lk,
                               start_pos, n_h, D_qk, D_v, k, scale, reinterpret_cast<__nv_bfloat16*>(out), lse,
                               vl ? vl->cu_q : nullptr, vl ? vl->cu_k : nullptr, vl ? vl->sp : nullptr);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("simt attention launch: ") + cudaGetErrorString(e));
    return DSA_OK;
  }
  return set_error(DSA_ERR_UNSUPPORTED,
                   "dsa_sparse_attn: supported shapes are MLA (128 heads, 576/512, K = V) or "
                   "n_h <= 128 with D_qk, D_v <= 128");
}

}  // namespace dsa
