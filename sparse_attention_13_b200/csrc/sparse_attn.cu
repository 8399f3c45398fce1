// sparse_attn.cu -- sparse core attention over the selected positions.
//
// "注意力机制中的 Index" §2 (alpha-hat / o-hat: softmax over exactly S_t, then
// the weighted sum of the selected values) and §4 (MLA: every query head reads
// the same latent row c_s; K = the 576-wide latent row, V = its first 512
// columns).
//
// mla_sparse_attn_kernel (n_h = 128, D_qk = 576, D_v = 512, K = V = latent):
//   A cluster of two CTAs owns one query row at a time.  CTA c holds half of
//   the query in TMEM (Q[:, 288c : 288c+288], the A operand of the QK UMMA) and
//   half of the output accumulator (O[:, 256c : 256c+256], fp32 in TMEM).
//   Per chunk of 64 selected rows:
//     producer warp  TMA gather4 of the chunk's latent rows, 5 slabs of 64
//                    columns each (CTA0 columns 0..319, CTA1 256..575),
//                    128B-swizzled, into a 3-stage ring;
//     MMA warp       S_c = Q_c K_c^T over the CTA's 288 columns (18 K16 UMMAs,
//                    A from TMEM), then, one chunk behind, O_c += P V_c with
//                    V_c the gathered slabs read as an MN-major B operand;
//     softmax warps  (thread = head = TMEM lane) read S_c, swap partial score
//                    tiles with the peer CTA through distributed shared memory
//                    (S = S_0 + S_1, identical in both CTAs because fp32
//                    addition commutes), mask padded rows, run the online
//                    softmax in the log2 domain with lazy rescaling of O
//                    (only when the running max grows by more than 2^8), and
//                    write P as bf16 into a double-buffered K-major tile.
//   The finished row is normalised by the softmax sum and stored as bf16.
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

// ------------------------------------------------------------------ SIMT
constexpr int kSimtThreads = 128;

__global__ void __launch_bounds__(kSimtThreads)
simt_sparse_attn_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kb,
                        int64_t ks, const __nv_bfloat16* __restrict__ vb, int64_t vs,
                        const int32_t* __restrict__ idx, int B, int Lq, int Lk, int start_pos,
                        int n_h, int Dqk, int Dv, int k, float scale, __nv_bfloat16* __restrict__ out,
                        float* __restrict__ lse) {
  extern __shared__ float qs[];  // [n_h][Dqk]
  const size_t row = blockIdx.x;
  const int b = static_cast<int>(row / Lq);
  const int i = static_cast<int>(row % Lq);
  const int T = start_pos + i;
  const int nv = min(T, k);
  for (int e = threadIdx.x; e < n_h * Dqk; e += kSimtThreads)
    qs[e] = __bfloat162float(q[row * n_h * Dqk + e]);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t* irow = idx + row * k;
  const __nv_bfloat16* kbase = kb + static_cast<int64_t>(b) * Lk * ks;
  const __nv_bfloat16* vbase = vb + static_cast<int64_t>(b) * Lk * vs;
  const float sl2 = scale * 1.4426950408889634f;
  for (int h = warp; h < n_h; h += kSimtThreads / 32) {
    float m = -INFINITY, l = 0.f;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int r = 0; r < nv; ++r) {
      const int s = irow[r];
      if (s < 0) continue;
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
constexpr int kSlabs = 5;                      // 64-column slabs gathered per CTA
constexpr int kSlabBytes = kChunk * 128;       // 8 KB
constexpr int kStageBytes = kSlabs * kSlabBytes;
constexpr int kStages = 3;
constexpr int kPBytes = kNH * 128;             // P tile [128 heads][64 rows] bf16
constexpr int kXBytes = kNH * kChunk * 4;      // partial score tile fp32
constexpr int kQSteps = 18;                    // 288 / 16
constexpr uint32_t kOCol = 0, kSCol = 256, kQCol = 320;
constexpr int kMlaThreads = 192;               // 4 softmax warps, producer, MMA
constexpr int kProdWarp = 4, kMmaWarpA = 5;
constexpr float kRescaleThresh = 8.0f;          // log2 units

struct MlaBars {
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full, s_free;
  uint64_t p_full[2], pv_done[2];
  uint64_t o_full, o_free, q_full;
  uint64_t x_full[2], x_free[2];
  unsigned long long kvmask[kStages];
  uint32_t tmem_slot;
  int abort_flag;
};

constexpr int kMlaSmem = 1024 + kStages * kStageBytes + 2 * kPBytes + 2 * kXBytes + 1024;

struct MlaParams {
  const __nv_bfloat16* q;   // [B*Lq][128][576]
  const int32_t* idx;       // [B*Lq][k]
  __nv_bfloat16* out;       // [B*Lq][128][512]
  float* lse;               // [B*Lq][128] or null
  unsigned int* err;
  int B, Lq, Lk, start_pos, k;
  float scale_log2;
};

__device__ __forceinline__ int item_chunks(const MlaParams& p, int item) {
  const int i = item % p.Lq;
  const int nv = min(p.start_pos + i, p.k);
  return (nv + kChunk - 1) / kChunk;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kMlaThreads, 1)
mla_sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_kv, const MlaParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* kv_smem = smem;
  uint8_t* p_smem = kv_smem + kStages * kStageBytes;
  uint8_t* x_smem = p_smem + 2 * kPBytes;
  MlaBars* bb = reinterpret_cast<MlaBars*>(x_smem + 2 * kXBytes);
  volatile int* abort_flag = &bb->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;
  const int n_items = p.B * p.Lq;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&bb->kv_full[s], 1); mbar_init(&bb->kv_empty[s], 1); }
    mbar_init(&bb->s_full, 1);
    mbar_init(&bb->s_free, 128);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bb->p_full[b], 128);
      mbar_init(&bb->pv_done[b], 1);
      mbar_init(&bb->x_full[b], 128);
      mbar_init(&bb->x_free[b], 128);
    }
    mbar_init(&bb->o_full, 1);
    mbar_init(&bb->o_free, 128);
    mbar_init(&bb->q_full, 128);
    bb->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarpA) {
    tmem_alloc(&bb->tmem_slot, 512);
    tmem_relinquish();
  }
  if (warp == kProdWarp && lane == 0) tma_prefetch_desc(&tm_kv);
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = bb->tmem_slot;

  if (warp == kProdWarp) {
    // ------------------------------------------------------------ gather
    uint32_t g = 0;  // global chunk counter
    bool ok = true;
    for (int item = pair; item < n_items && ok; item += n_pairs) {
      const int nch = item_chunks(p, item);
      const int b = item / p.Lq;
      const int i = item % p.Lq;
      const int nv = min(p.start_pos + i, p.k);
      const int32_t* irow = p.idx + static_cast<size_t>(item) * p.k;
      for (int c = 0; c < nch; ++c, ++g) {
        const int stage = g % kStages;
        const uint32_t ph = (g / kStages) & 1;
        if (!mbar_wait(&bb->kv_empty[stage], ph ^ 1, abort_flag)) { ok = false; break; }
        const int r0 = c * kChunk + lane, r1 = r0 + 32;
        const int s0 = r0 < nv ? irow[r0] : -1;
        const int s1 = r1 < nv ? irow[r1] : -1;
        const bool v0 = s0 >= 0 && s0 < p.Lk, v1 = s1 >= 0 && s1 < p.Lk;
        const int row0 = b * p.Lk + (v0 ? s0 : 0);
        const int row1 = b * p.Lk + (v1 ? s1 : 0);
        const unsigned m0 = __ballot_sync(0xffffffffu, v0);
        const unsigned m1 = __ballot_sync(0xffffffffu, v1);
        if (lane == 0) {
          bb->kvmask[stage] = static_cast<unsigned long long>(m0) | (static_cast<unsigned long long>(m1) << 32);
          mbar_arrive_expect_tx(&bb->kv_full[stage], kStageBytes);
        }
        uint8_t* dst = kv_smem + stage * kStageBytes;
        const int col0 = rank == 0 ? 0 : 256;
#pragma unroll
        for (int grp = 0; grp < 16; ++grp) {
          const int src = (grp & 7) * 4;
          const int a0 = __shfl_sync(0xffffffffu, grp < 8 ? row0 : row1, src + 0);
          const int a1 = __shfl_sync(0xffffffffu, grp < 8 ? row0 : row1, src + 1);
          const int a2 = __shfl_sync(0xffffffffu, grp < 8 ? row0 : row1, src + 2);
          const int a3 = __shfl_sync(0xffffffffu, grp < 8 ? row0 : row1, src + 3);
          if (lane == 0) {
#pragma unroll
            for (int sl = 0; sl < kSlabs; ++sl)
              tma_gather4(dst + sl * kSlabBytes + grp * 512, &tm_kv, &bb->kv_full[stage],
                          col0 + sl * 64, a0, a1, a2, a3);
          }
        }
      }
    }
  } else if (warp == kMmaWarpA) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      uint32_t g = 0, it_n = 0;
      bool ok = true;
      const uint32_t idesc_qk = make_idesc_bf16(128, kChunk, 0, 0);
      const uint32_t idesc_pv = make_idesc_bf16(128, 256, 0, 1);
      auto issue_pv = [&](uint32_t gc, bool first) -> bool {
        const int pb = gc & 1;
        if (!mbar_wait(&bb->p_full[pb], (gc >> 1) & 1, abort_flag)) return false;
        tc_fence_after();
        const int stage = gc % kStages;
        // V = this CTA's slabs 0..3: value columns 0..255 (CTA0) or 256..511 (CTA1)
        const uint32_t v_base = smem_u32(kv_smem + stage * kStageBytes);
        const uint32_t a_base = smem_u32(p_smem + pb * kPBytes);
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk) {
          const uint64_t ad = make_smem_desc(a_base + kk * 32, 16, 1024, kSwizzle128B);
          const uint64_t bd = make_smem_desc(v_base + kk * 2048, kSlabBytes, 1024, kSwizzle128B);
          umma_bf16_ss(tmem + kOCol, ad, bd, idesc_pv, (first && kk == 0) ? 0u : 1u);
        }
        umma_commit(&bb->pv_done[pb]);
        umma_commit(&bb->kv_empty[stage]);
        return true;
      };
      for (int item = pair; item < n_items && ok; item += n_pairs) {
        const int nch = item_chunks(p, item);
        if (nch == 0) continue;
        if (!mbar_wait(&bb->q_full, it_n & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        for (int c = 0; c < nch && ok; ++c, ++g) {
          const int stage = g % kStages;
          if (!mbar_wait(&bb->kv_full[stage], (g / kStages) & 1, abort_flag)) { ok = false; break; }
          if (!mbar_wait(&bb->s_free, (g & 1) ^ 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kb = smem_u32(kv_smem + stage * kStageBytes);
#pragma unroll
          for (int st = 0; st < kQSteps; ++st) {
            // CTA0: slabs 0..3 + first half of slab 4; CTA1: second half of slab 0 + slabs 1..4
            const int e = rank == 0 ? st : st + 2;
            const uint64_t bd = make_smem_desc(kb + (e >> 2) * kSlabBytes + (e & 3) * 32, 16, 1024,
                                               kSwizzle128B);
            umma_bf16_ts(tmem + kSCol, tmem + kQCol + st * 8, bd, idesc_qk, st != 0);
          }
          umma_commit(&bb->s_full);
          if (c >= 1) {
            if (c == 1 && !mbar_wait(&bb->o_free, (it_n & 1) ^ 1, abort_flag)) { ok = false; break; }
            if (!issue_pv(g - 1, c == 1)) { ok = false; break; }
          }
        }
        if (!ok) break;
        if (nch == 1 && !mbar_wait(&bb->o_free, (it_n & 1) ^ 1, abort_flag)) { ok = false; break; }
        if (!issue_pv(g - 1, nch == 1)) { ok = false; break; }
        umma_commit(&bb->o_full);
        ++it_n;
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int h = threadIdx.x;  // head = TMEM lane
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const uint32_t x_local = smem_u32(x_smem);
    const uint32_t x_remote = mapa_shared(x_local, peer);
    const uint32_t xfull_remote[2] = {mapa_shared(smem_u32(&bb->x_full[0]), peer),
                                      mapa_shared(smem_u32(&bb->x_full[1]), peer)};
    const uint32_t xfree_remote[2] = {mapa_shared(smem_u32(&bb->x_free[0]), peer),
                                      mapa_shared(smem_u32(&bb->x_free[1]), peer)};
    uint32_t g = 0, it_n = 0;
    bool ok = true;
    for (int item = pair; item < n_items && ok; item += n_pairs) {
      const int nch = item_chunks(p, item);
      const size_t row = static_cast<size_t>(item);
      __nv_bfloat16* orow = p.out + (row * kNH + h) * kDV + rank * 256;
      if (nch == 0) {
        const uint4 z = make_uint4(0, 0, 0, 0);
        for (int j = 0; j < 32; ++j) reinterpret_cast<uint4*>(orow)[j] = z;
        if (p.lse && rank == 0) p.lse[row * kNH + h] = -INFINITY;
        continue;
      }
      // this CTA's half of the query row -> TMEM (A operand of QK)
      {
        const uint4* qsrc = reinterpret_cast<const uint4*>(p.q + (row * kNH + h) * kDQK + rank * 288);
#pragma unroll
        for (int blk = 0; blk < 5; ++blk) {
          uint32_t r[32];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            uint4 v = make_uint4(0, 0, 0, 0);
            if (blk * 8 + j < 36) v = __ldg(qsrc + blk * 8 + j);
            r[4 * j] = v.x; r[4 * j + 1] = v.y; r[4 * j + 2] = v.z; r[4 * j + 3] = v.w;
          }
          tmem_st32x32(t_lane + kQCol + blk * 32, r);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bb->q_full);
      }
      // l_run: sum of the bf16 weights that PV multiplies (normalises O);
      // l_lse: the same sum in fp32 before rounding (for the log-sum-exp).
      float m_run = -INFINITY, l_run = 0.f, l_lse = 0.f;
      for (int c = 0; c < nch; ++c, ++g) {
        const int stage = g % kStages;
        const int xb = g & 1;
        if (!mbar_wait(&bb->s_full, g & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        float s[64];
        {
          uint32_t v[32];
          tmem_ld32<32>(t_lane + kSCol, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) s[j] = __uint_as_float(v[j]);
          tmem_ld32<32>(t_lane + kSCol + 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) s[32 + j] = __uint_as_float(v[j]);
        }
        tc_fence_before();
        mbar_arrive(&bb->s_free);
        // swap partial scores with the peer: my partial -> peer's buffer xb
        if (!mbar_wait_cluster(&bb->x_free[xb], ((g >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
        {
          const uint32_t rowbase = x_remote + xb * kXBytes + h * 256;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            st_cluster_v4(rowbase + ((j ^ (h & 15)) << 4), s[4 * j], s[4 * j + 1], s[4 * j + 2],
                          s[4 * j + 3]);
        }
        mbar_arrive_remote(xfull_remote[xb]);
        if (!mbar_wait_cluster(&bb->x_full[xb], (g >> 1) & 1, abort_flag)) { ok = false; break; }
        {
          const float4* xr = reinterpret_cast<const float4*>(x_smem + xb * kXBytes + h * 256);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float4 o = xr[j ^ (h & 15)];
            s[4 * j] += o.x; s[4 * j + 1] += o.y; s[4 * j + 2] += o.z; s[4 * j + 3] += o.w;
          }
        }
        mbar_arrive_remote(xfree_remote[xb]);
        // online softmax over this chunk (log2 domain), lazy rescale
        if (!mbar_wait(&bb->kv_full[stage], (g / kStages) & 1, abort_flag)) { ok = false; break; }
        const unsigned long long vmask = bb->kvmask[stage];
        float cmax = -INFINITY;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          s[j] = ((vmask >> j) & 1ull) ? s[j] * p.scale_log2 : -INFINITY;
          cmax = fmaxf(cmax, s[j]);
        }
        if (cmax > m_run + kRescaleThresh) {
          const float factor = exp2f(m_run - cmax);  // 0 when m_run = -inf
          if (c > 0) {
            // O holds PV(0..c-1): wait for PV(c-1), then scale it in place
            if (!mbar_wait(&bb->pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
#pragma unroll 1
            for (int blk = 0; blk < 8; ++blk) {
              uint32_t v[32];
              tmem_ld32<32>(t_lane + kOCol + blk * 32, v);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * factor);
              tmem_st32x32(t_lane + kOCol + blk * 32, v);
            }
            tmem_st_wait();
          }
          l_run *= factor;
          l_lse *= factor;
          m_run = cmax;
        }
        float psum = 0.f, esum = 0.f;
        uint32_t pk[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float a = m_run == -INFINITY ? 0.f : exp2f(s[2 * j] - m_run);
          const float bq = m_run == -INFINITY ? 0.f : exp2f(s[2 * j + 1] - m_run);
          const __nv_bfloat162 pr = __floats2bfloat162_rn(a, bq);
          const float2 pf = __bfloat1622float2(pr);
          psum += pf.x + pf.y;
          esum += a + bq;
          pk[j] = *reinterpret_cast<const uint32_t*>(&pr);
        }
        l_run += psum;
        l_lse += esum;
        // P buffer xb was last read by PV(g-2)
        if (g >= 2 && !mbar_wait(&bb->pv_done[xb], ((g - 2) >> 1) & 1, abort_flag)) { ok = false; break; }
        {
          uint8_t* prow = p_smem + xb * kPBytes + h * 128;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4*>(prow + ((j ^ (h & 7)) << 4)) =
                make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bb->p_full[xb]);
      }
      if (!ok) break;
      // epilogue: O / l -> bf16
      if (!mbar_wait(&bb->o_full, it_n & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll 1
      for (int blk = 0; blk < 8; ++blk) {
        uint32_t v[32];
        tmem_ld32<32>(t_lane + kOCol + blk * 32, v);
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
      tc_fence_before();
      mbar_arrive(&bb->o_free);
      if (p.lse && rank == 0)
        p.lse[row * kNH + h] = l_lse > 0.f ? (m_run + log2f(l_lse)) * 0.6931471805599453f : -INFINITY;
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

}  // namespace

size_t sparse_attn_ws_bytes(int, int, int, int, int) { return 0; }

dsa_status sparse_attn_launch(const dsa_bf16* q, const dsa_bf16* kbuf, int64_t k_row_stride,
                              const dsa_bf16* vbuf, int64_t v_row_stride, const int32_t* idx,
                              int B, int Lq, int Lk, int start_pos, int n_h, int D_qk, int D_v,
                              int k, float scale, dsa_bf16* out, float* lse, void* ws,
                              size_t ws_bytes, cudaStream_t stream) {
  (void)ws;
  (void)ws_bytes;
  const long long rows = static_cast<long long>(B) * Lq;
  if (rows > (1ll << 31) - 1) return set_error(DSA_ERR_UNSUPPORTED, "dsa_sparse_attn: too many rows");
  const bool mla = n_h == kNH && D_qk == kDQK && D_v == kDV && kbuf == vbuf &&
                   k_row_stride == v_row_stride;
  if (mla) {
    CUtensorMap tkv;
    if (!encode_tiled_2d(&tkv, kbuf, kDQK, static_cast<uint64_t>(B) * Lk,
                         static_cast<uint64_t>(k_row_stride) * 2, 64, 1, CU_TENSOR_MAP_SWIZZLE_128B))
      return set_error(DSA_ERR_CUDA, "tensor map for the latent cache failed");
    MlaParams p{};
    p.q = reinterpret_cast<const __nv_bfloat16*>(q);
    p.idx = idx;
    p.out = reinterpret_cast<__nv_bfloat16*>(out);
    p.lse = lse;
    p.err = device_error_word();
    if (!p.err) return set_error(DSA_ERR_CUDA, "cannot resolve the device error word");
    p.B = B; p.Lq = Lq; p.Lk = Lk; p.start_pos = start_pos; p.k = k;
    p.scale_log2 = scale * 1.4426950408889634f;
    const int sms = device_sm_count();
    if (sms <= 0) return set_error(DSA_ERR_CUDA, "cannot query the device SM count");
    const long long pairs = std::min<long long>(rows, sms / 2);
    cudaError_t e = cudaFuncSetAttribute(mla_sparse_attn_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kMlaSmem);
    if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("mla smem attribute: ") + cudaGetErrorString(e));
    mla_sparse_attn_kernel<<<static_cast<unsigned>(2 * pairs), kMlaThreads, kMlaSmem, stream>>>(tkv, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("mla launch: ") + cudaGetErrorString(e));
    return DSA_OK;
  }
  if (n_h <= 128 && D_qk <= 128 && D_v <= 128) {
    const int smem = n_h * D_qk * 4;
    if (smem > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(simt_sparse_attn_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("simt smem attribute: ") + cudaGetErrorString(e));
    }
    simt_sparse_attn_kernel<<<static_cast<unsigned>(rows), kSimtThreads, smem, stream>>>(
        reinterpret_cast<const __nv_bfloat16*>(q), reinterpret_cast<const __nv_bfloat16*>(kbuf),
        k_row_stride, reinterpret_cast<const __nv_bfloat16*>(vbuf), v_row_stride, idx, B, Lq, Lk,
        start_pos, n_h, D_qk, D_v, k, scale, reinterpret_cast<__nv_bfloat16*>(out), lse);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("simt attention launch: ") + cudaGetErrorString(e));
    return DSA_OK;
  }
  return set_error(DSA_ERR_UNSUPPORTED,
                   "dsa_sparse_attn: supported shapes are MLA (128 heads, 576/512, K = V) or "
                   "n_h <= 128 with D_qk, D_v <= 128");
}

}  // namespace dsa
