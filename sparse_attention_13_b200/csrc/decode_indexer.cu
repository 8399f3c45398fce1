// decode_indexer.cu -- lightning indexer + top-k for one query row per
// sequence against a long cache (decode).
//
// Same operation as indexer_topk.cu ("注意力机制中的 Index" §4: I[t,s] =
// sum_j w[t,j] ReLU(q[t,j].k[s]) over s < t, TopK with ties to the lower
// position, ascending output, -1 padding), organised for the decode shape
// where reading the key cache from HBM is the cost and a row of scores is
// small enough to keep:
//   decode_score_kernel  one CTA per (sequence, key range): TMA streams
//        128-key tiles through a 6-stage ring, one thread issues a
//        128 x H_I x d_I UMMA per tile into a 4-deep TMEM ring, four
//        epilogue warps (thread = key) apply ReLU and w and store each score
//        as an order-preserving 32-bit key.
//   decode_topk_kernel   one 8-CTA cluster per sequence: each CTA holds 1/8 of
//        the row's keys in shared memory; an MSB-first radix select (8-bit
//        digits) sums the CTAs' histograms through distributed shared memory;
//        keys equal to the threshold are taken in position order; each CTA
//        then writes its selected positions at its offset in the row.
#include <cuda_bf16.h>

#include <algorithm>

#include "dsa_internal.h"
#include "dsa_ptx.cuh"

namespace dsa {
namespace {

constexpr int kTile = 128;          // keys per tile = UMMA M
constexpr int kDecStages = 6;
constexpr int kDecBufs = 4;         // TMEM accumulators of 64 columns
constexpr int kDecThreads = 192;    // 4 epilogue warps, TMA warp, MMA warp
constexpr int kDecTmaWarp = 4, kDecMmaWarp = 5;
constexpr int kClusterRanks = 8;
constexpr int kTopkThreads = 1024;
constexpr int kMaxSlice = 48 * 1024;  // keys per CTA slice (192 KB)

template <int H, int D>
struct DecCfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kQChunkBytes = H * 128;
  static constexpr int kQBytes = kChunks * kQChunkBytes;
  static constexpr int kKeyChunkBytes = kTile * 128;
  static constexpr int kStageBytes = kTile * D * 2;
};

struct DecParams {
  const float* w;        // [B][H]
  uint32_t* keys;        // [B][Lk] score keys
  unsigned int* err;
  int B, Lk, T, n_split, split_len;
};

template <int H, int D>
__global__ void __launch_bounds__(kDecThreads, 1)
decode_score_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const DecParams p) {
  using C = DecCfg<H, D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* q_smem = smem;
  uint8_t* key_smem = q_smem + ((C::kQBytes + 1023) / 1024) * 1024;
  uint64_t* bars = reinterpret_cast<uint64_t*>(key_smem + kDecStages * C::kStageBytes);
  uint64_t* key_full = bars;
  uint64_t* key_empty = bars + kDecStages;
  uint64_t* t_full = key_empty + kDecStages;
  uint64_t* t_empty = t_full + kDecBufs;
  uint64_t* q_full = t_empty + kDecBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* w_smem = reinterpret_cast<float*>(tmem_slot + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x / p.n_split;
  const int sp = blockIdx.x % p.n_split;
  const int s_begin = sp * p.split_len;
  const int s_end = min(p.T, s_begin + p.split_len);
  const int n_tiles = s_end > s_begin ? (s_end - s_begin + kTile - 1) / kTile : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) { mbar_init(&key_full[s], 1); mbar_init(&key_empty[s], 1); }
    for (int j = 0; j < kDecBufs; ++j) { mbar_init(&t_full[j], 1); mbar_init(&t_empty[j], 4); }
    mbar_init(q_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (threadIdx.x < H) w_smem[threadIdx.x] = p.w[static_cast<size_t>(b) * H + threadIdx.x];
  if (warp == kDecMmaWarp) {
    tmem_alloc(tmem_slot, kDecBufs * 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kDecTmaWarp) {
    if (lane == 0 && n_tiles > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      mbar_arrive_expect_tx(q_full, C::kQBytes);
      for (int c = 0; c < C::kChunks; ++c)
        tma_load_3d(q_smem + c * C::kQChunkBytes, &tm_q, q_full, c * 64, 0, b);
      for (int t = 0; t < n_tiles; ++t) {
        const int stage = t % kDecStages;
        if (!mbar_wait(&key_empty[stage], ((t / kDecStages) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&key_full[stage], C::kStageBytes);
        uint8_t* dst = key_smem + stage * C::kStageBytes;
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_3d(dst + c * C::kKeyChunkBytes, &tm_k, &key_full[stage], c * 64, s_begin + t * kTile, b);
      }
    }
  } else if (warp == kDecMmaWarp) {
    if (lane == 0 && n_tiles > 0) {
      const uint32_t idesc = make_idesc_bf16(128, H, 0, 0);
      bool ok = mbar_wait(q_full, 0, abort_flag);
      tc_fence_after();
      for (int t = 0; t < n_tiles && ok; ++t) {
        const int stage = t % kDecStages, buf = t % kDecBufs;
        if (!mbar_wait(&key_full[stage], (t / kDecStages) & 1, abort_flag)) break;
        if (!mbar_wait(&t_empty[buf], ((t / kDecBufs) & 1) ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(key_smem + stage * C::kStageBytes);
        const uint32_t b_base = smem_u32(q_smem);
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = make_smem_desc(a_base + c * C::kKeyChunkBytes + kk * 32, 16, 1024, kSwizzle128B);
            const uint64_t bd = make_smem_desc(b_base + c * C::kQChunkBytes + kk * 32, 16, 1024, kSwizzle128B);
            umma_bf16_ss(tmem + buf * 64, ad, bd, idesc, (c | kk) != 0);
          }
        umma_commit(&t_full[buf]);
        umma_commit(&key_empty[stage]);
      }
    }
  } else {
    // epilogue: thread = key (TMEM lane 32*warp + lane)
    float w[H];
#pragma unroll
    for (int j = 0; j < H; ++j) w[j] = w_smem[j];
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    uint32_t* out = p.keys + static_cast<size_t>(b) * p.Lk;
    for (int t = 0; t < n_tiles; ++t) {
      const int buf = t % kDecBufs;
      if (!mbar_wait(&t_full[buf], (t / kDecBufs) & 1, abort_flag)) break;
      tc_fence_after();
      uint32_t v[H];
      if constexpr (H >= 32) {
#pragma unroll
        for (int c = 0; c < H / 32; ++c)
          tmem_ld32<32>(t_lane + buf * 64 + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&v[c * 32]));
      } else {
        tmem_ld32<H>(t_lane + buf * 64, v);
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&t_empty[buf]);
      // heads j = 4i + r accumulate into a[r]; combined as (a0 + a1) + (a2 + a3)
      float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < H; ++j) a[j & 3] = fmaf(fmaxf(__uint_as_float(v[j]), 0.f), w[j], a[j & 3]);
      const float score = (a[0] + a[1]) + (a[2] + a[3]);
      const int s = s_begin + t * kTile + warp * 32 + lane;
      if (s < s_end) out[s] = float_key(score);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) atomicOr(p.err, 1u);
  if (warp == kDecMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kDecBufs * 64);
  }
}

__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t cluster_addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
  return v;
}

__device__ __forceinline__ int block_scan_excl(int x, int* ws, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) ws[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int v = ws[lane];
    int vi = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, vi, o);
      if (lane >= o) vi += y;
    }
    ws[lane] = vi - v;
    if (lane == 31) ws[32] = vi;
  }
  __syncthreads();
  const int r = ws[warp] + incl - x;
  total = ws[32];
  __syncthreads();
  return r;
}

struct TopkShared {
  int hist[256];
  int tot[256];
  int scan_ws[33];
  int sel_bin, kk_new, bin_count;
  int n_gt, n_tie;
};

__global__ void __cluster_dims__(kClusterRanks, 1, 1) __launch_bounds__(kTopkThreads, 1)
decode_topk_kernel(const uint32_t* __restrict__ keys, int32_t* __restrict__ idx, int Lk, int T, int k) {
  extern __shared__ uint32_t slice[];
  __shared__ TopkShared sh;
  const int tid = threadIdx.x;
  const uint32_t rank = cluster_ctarank();
  const size_t row = blockIdx.x / kClusterRanks;
  const int per = (T + kClusterRanks - 1) / kClusterRanks;
  const int lo = min(T, static_cast<int>(rank) * per);
  const int n = min(T, lo + per) - lo;
  const uint32_t* src = keys + row * Lk + lo;
  for (int e = tid; e < n; e += kTopkThreads) slice[e] = src[e];
  __syncthreads();
  uint32_t thr = 0u;
  int ties = 1 << 30;
  if (T > k) {
    uint32_t prefix = 0u;
    int kk = k;
    bool exact = true;
    for (int shift = 24; shift >= 0; shift -= 8) {
      if (tid < 256) sh.hist[tid] = 0;
      __syncthreads();
      // warp-aggregated: scores cluster in a few bins, so one atomic per
      // distinct bin and warp instead of one per key
      for (int base = (tid & ~31); base < n; base += kTopkThreads) {
        const int e = base + (tid & 31);
        uint32_t bin = 256u;
        if (e < n) {
          const uint32_t key = slice[e];
          if (shift == 24 || (key >> (shift + 8)) == (prefix >> (shift + 8))) bin = (key >> shift) & 255u;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        if (bin < 256u && (tid & 31) == __ffs(peers) - 1) atomicAdd(&sh.hist[bin], __popc(peers));
      }
      cluster_sync();  // every CTA's histogram is complete
      if (tid < 256) {
        const uint32_t a = smem_u32(&sh.hist[tid]);
        int sum = 0;
#pragma unroll
        for (int r = 0; r < kClusterRanks; ++r) sum += static_cast<int>(ld_cluster_u32(mapa_shared(a, r)));
        sh.tot[tid] = sum;
      }
      __syncthreads();
      if (tid < 32) {
        int loc[8];
        int sum = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) { loc[i] = sh.tot[tid * 8 + i]; sum += loc[i]; }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_down_sync(0xffffffffu, incl, o);
          if (tid + o < 32) incl += y;
        }
        int above = incl - sum;
#pragma unroll
        for (int i = 7; i >= 0; --i) {
          if (above < kk && above + loc[i] >= kk) {
            sh.sel_bin = tid * 8 + i;
            sh.kk_new = kk - above;
            sh.bin_count = loc[i];
          }
          above += loc[i];
        }
      }
      cluster_sync();  // peers finished reading this CTA's histogram
      prefix |= static_cast<uint32_t>(sh.sel_bin) << shift;
      kk = sh.kk_new;
      if (sh.bin_count == kk) {
        exact = false;
        break;
      }
    }
    thr = prefix;
    if (exact) ties = kk;
  }
  const bool limited = ties < (1 << 30);
  // this CTA's counts of keys above the threshold and equal to it
  const int seg = (n + kTopkThreads - 1) / kTopkThreads;
  const int e0 = min(n, tid * seg), e1 = min(n, e0 + seg);
  int my_gt = 0, my_tie = 0;
  for (int e = e0; e < e1; ++e) {
    const uint32_t key = slice[e];
    if (limited) {
      my_gt += key > thr;
      my_tie += key == thr;
    } else {
      my_gt += key >= thr;
    }
  }
  int tot_gt, tot_tie;
  const int gt_base = block_scan_excl(my_gt, sh.scan_ws, tot_gt);
  const int tie_base = block_scan_excl(my_tie, sh.scan_ws, tot_tie);
  if (tid == 0) { sh.n_gt = tot_gt; sh.n_tie = tot_tie; }
  cluster_sync();
  // offsets of this CTA among the cluster (positions are ascending across ranks)
  int out_base = 0, cta_tie_base = 0;
  {
    const uint32_t a_gt = smem_u32(&sh.n_gt), a_tie = smem_u32(&sh.n_tie);
    int tb = 0;
    for (uint32_t r = 0; r < rank; ++r) {
      const int g = static_cast<int>(ld_cluster_u32(mapa_shared(a_gt, r)));
      const int tc = static_cast<int>(ld_cluster_u32(mapa_shared(a_tie, r)));
      const int take = limited ? max(0, min(tc, ties - tb)) : 0;
      out_base += g + take;
      tb += tc;
    }
    cta_tie_base = tb;
  }
  // thread offsets: keys above thr, plus ties whose global rank is < ties
  int my_take = 0;
  if (limited) {
    const int t0 = cta_tie_base + tie_base;
    my_take = max(0, min(my_tie, ties - t0));
  }
  int tot_keep;
  const int pos0 = block_scan_excl(my_gt + my_take, sh.scan_ws, tot_keep);
  (void)gt_base;
  int32_t* out = idx + row * k;
  {
    int pos = out_base + pos0;
    int tr = cta_tie_base + tie_base;
    for (int e = e0; e < e1; ++e) {
      const uint32_t key = slice[e];
      bool kp;
      if (limited) {
        kp = key > thr || (key == thr && tr < ties);
        tr += key == thr;
      } else {
        kp = key >= thr;
      }
      if (kp) {
        if (pos < k) out[pos] = lo + e;
        ++pos;
      }
    }
  }
  // padding when fewer than k positions are visible
  if (rank == kClusterRanks - 1) {
    const int total = out_base + tot_keep;
    for (int q = total + tid; q < k; q += kTopkThreads) out[q] = -1;
  }
  cluster_sync();  // no CTA leaves while peers may read its shared memory
}

template <int H, int D>
dsa_status launch_dec(const CUtensorMap& tq, const CUtensorMap& tk, const DecParams& p, int grid,
                      cudaStream_t stream) {
  using C = DecCfg<H, D>;
  const int smem = 1024 + ((C::kQBytes + 1023) / 1024) * 1024 + kDecStages * C::kStageBytes + 512 + H * 4;
  auto kern = decode_score_kernel<H, D>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("decode score smem attribute: ") + cudaGetErrorString(e));
  kern<<<grid, kDecThreads, smem, stream>>>(tq, tk, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("decode score launch: ") + cudaGetErrorString(e));
  return DSA_OK;
}

}  // namespace

bool decode_indexer_applies(int Lq, int Lk, int start_pos, int H, int d) {
  const int T = start_pos;  // the single query row sits at t = start_pos
  return Lq == 1 && (H == 16 || H == 32 || H == 64) && (d == 64 || d == 128) && T >= 1 &&
         (T + kClusterRanks - 1) / kClusterRanks <= kMaxSlice && Lk >= T;
}

size_t decode_indexer_ws_bytes(int B, int Lk) {
  return ((static_cast<size_t>(B) * Lk * 4 + 255) / 256) * 256;
}

dsa_status decode_indexer_launch(const dsa_bf16* q_idx, const dsa_bf16* k_idx, const float* w, int B,
                                 int Lk, int start_pos, int H, int d, int k, int32_t* idx, void* ws,
                                 size_t ws_bytes, cudaStream_t stream) {
  const int T = start_pos;
  if (ws_bytes < decode_indexer_ws_bytes(B, Lk)) return set_error(DSA_ERR_WORKSPACE, "indexer workspace too small");
  const int sms = device_sm_count();
  if (sms <= 0) return set_error(DSA_ERR_CUDA, "cannot query the device SM count");
  const int tiles = (T + kTile - 1) / kTile;
  const int n_split = std::max(1, std::min(tiles, sms / B > 0 ? sms / B : 1));
  DecParams p{};
  p.w = w;
  p.keys = static_cast<uint32_t*>(ws);
  p.err = device_error_word();
  if (!p.err) return set_error(DSA_ERR_CUDA, "cannot resolve the device error word");
  p.B = B; p.Lk = Lk; p.T = T; p.n_split = n_split;
  p.split_len = ((tiles + n_split - 1) / n_split) * kTile;
  CUtensorMap tq, tk;
  if (!encode_tiled_3d(&tq, q_idx, d, H, B, static_cast<uint64_t>(d) * 2, static_cast<uint64_t>(H) * d * 2,
                       64, H, CU_TENSOR_MAP_SWIZZLE_128B))
    return set_error(DSA_ERR_CUDA, "tensor map for q_idx failed");
  if (!encode_tiled_3d(&tk, k_idx, d, Lk, B, static_cast<uint64_t>(d) * 2, static_cast<uint64_t>(Lk) * d * 2,
                       64, kTile, CU_TENSOR_MAP_SWIZZLE_128B))
    return set_error(DSA_ERR_CUDA, "tensor map for k_idx failed");
  const int grid = B * n_split;
  dsa_status st = DSA_ERR_UNSUPPORTED;
  if (H == 16 && d == 64) st = launch_dec<16, 64>(tq, tk, p, grid, stream);
  if (H == 16 && d == 128) st = launch_dec<16, 128>(tq, tk, p, grid, stream);
  if (H == 32 && d == 64) st = launch_dec<32, 64>(tq, tk, p, grid, stream);
  if (H == 32 && d == 128) st = launch_dec<32, 128>(tq, tk, p, grid, stream);
  if (H == 64 && d == 64) st = launch_dec<64, 64>(tq, tk, p, grid, stream);
  if (H == 64 && d == 128) st = launch_dec<64, 128>(tq, tk, p, grid, stream);
  if (st != DSA_OK) return st;
  const int per = (T + kClusterRanks - 1) / kClusterRanks;
  const int tsmem = per * 4;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(decode_topk_kernel), std::max(tsmem, 1));
  if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("decode top-k smem attribute: ") + cudaGetErrorString(e));
  decode_topk_kernel<<<B * kClusterRanks, kTopkThreads, tsmem, stream>>>(p.keys, idx, Lk, T, k);
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("decode top-k launch: ") + cudaGetErrorString(e));
  return DSA_OK;
}

}  // namespace dsa
