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
//        epilogue warps (thread = key) apply ReLU and w, store each score as
//        an order-preserving 32-bit key and count it in a 4096-bin histogram
//        of the key's top 12 bits (written out per CTA at the end).
//   decode_topk_kernel   one 8-CTA cluster per sequence: each CTA holds 1/8 of
//        the row's keys in shared memory (one bulk copy).  The score
//        histograms, summed over the cluster through distributed shared
//        memory, give the 12-bit bin of the k-th key; keys above it are kept,
//        keys inside it go to a short candidate list.  Every CTA gathers the
//        whole cluster's lists and finds the exact k-th key by two more 10-bit
//        radix passes on its own.  Kept and tied positions are marked in
//        bitmaps, ties are granted in position order, and each CTA writes its
//        positions at its offset in the row.
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
constexpr int kHistBins = 4096;     // top 12 bits of the score key
constexpr int kHistShift = 20;
constexpr int kClusterRanks = 8;
constexpr int kPortion = kHistBins / kClusterRanks;  // bins reduced per CTA
constexpr int kTopkThreads = 1024;
constexpr int kMaxSlice = 40 * 1024;                  // keys per CTA slice
constexpr int kMaxWords = kMaxSlice / 32;
constexpr int kListCap = 4096;                        // candidates per CTA
constexpr int kMaxScoreCtasPerRow = 160;
constexpr int kSmemLimit = 227 * 1024;

__host__ __device__ constexpr int round_up(int x, int m) { return (x + m - 1) / m * m; }

template <int H, int D>
struct DecCfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kQChunkBytes = H * 128;
  static constexpr int kQBytes = kChunks * kQChunkBytes;
  static constexpr int kKeyChunkBytes = kTile * 128;
  static constexpr int kStageBytes = kTile * D * 2;
  static constexpr int kQAlloc = (kQBytes + 1023) / 1024 * 1024;
  static constexpr int kBarBytes = 256;
  static constexpr int kSmem = 1024 + kQAlloc + kDecStages * kStageBytes + kBarBytes + kHistBins * 4;
  static_assert(kSmem <= kSmemLimit, "decode score kernel shared memory");
};

struct DecParams {
  const float* w;        // [B][H]
  uint32_t* keys;        // [B][row_stride] score keys
  int* hist;             // [B][n_split][4096] per-CTA key histograms
  unsigned int* err;
  // Variable-length batches (both null for a uniform batch): sequence b's
  // row sits at t = sp[b] (at most T) and its keys are rows cu_k[b] ... of
  // the packed key tensor.
  const int* sp;
  const int* cu_k;
  int B, row_stride, T, n_split, split_len;
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
  uint8_t* key_smem = q_smem + C::kQAlloc;
  uint64_t* bars = reinterpret_cast<uint64_t*>(key_smem + kDecStages * C::kStageBytes);
  uint64_t* key_full = bars;
  uint64_t* key_empty = bars + kDecStages;
  uint64_t* t_full = key_empty + kDecStages;
  uint64_t* t_empty = t_full + kDecBufs;
  uint64_t* q_full = t_empty + kDecBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* hist_smem = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(bars) + C::kBarBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x / p.n_split;
  const int sp = blockIdx.x % p.n_split;
  const int s_begin = sp * p.split_len;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) { mbar_init(&key_full[s], 1); mbar_init(&key_empty[s], 1); }
    for (int j = 0; j < kDecBufs; ++j) { mbar_init(&t_full[j], 1); mbar_init(&t_empty[j], 4); }
    mbar_init(q_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  for (int i = threadIdx.x; i < kHistBins; i += kDecThreads) hist_smem[i] = 0;
  if (warp == kDecMmaWarp) {
    tmem_alloc(tmem_slot, kDecBufs * 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();
  pdl_wait();
  // the row's visible keys (per sequence when varlen; read after the wait,
  // since earlier work in the stream may write the positions)
  const int T = p.sp ? min(max(__ldg(p.sp + b), 0), p.T) : p.T;
  const int k_row0 = p.cu_k ? __ldg(p.cu_k + b) : 0;
  const int tb = p.cu_k ? 0 : b;
  const int s_end = min(T, s_begin + p.split_len);
  const int n_tiles = s_end > s_begin ? (s_end - s_begin + kTile - 1) / kTile : 0;

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
          tma_load_3d(dst + c * C::kKeyChunkBytes, &tm_k, &key_full[stage], c * 64, k_row0 + s_begin + t * kTile, tb);
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
    for (int j = 0; j < H; ++j) w[j] = __ldg(p.w + static_cast<size_t>(b) * H + j);
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    uint32_t* out = p.keys + static_cast<size_t>(b) * p.row_stride;
    for (int t = 0; t < n_tiles; ++t) {
      const int buf = t % kDecBufs;
      if (!__all_sync(0xffffffffu, mbar_wait(&t_full[buf], (t / kDecBufs) & 1, abort_flag))) break;
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
      if (s < s_end) {
        const uint32_t key = float_key(score);
        out[s] = key;
        atomicAdd(&hist_smem[key >> kHistShift], 1);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) atomicOr(p.err, 1u);
  if (warp == kDecMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kDecBufs * 64);
  }
  int4* hg = reinterpret_cast<int4*>(p.hist + static_cast<size_t>(blockIdx.x) * kHistBins);
  const int4* hs = reinterpret_cast<const int4*>(hist_smem);
  for (int i = threadIdx.x; i < kHistBins / 4; i += kDecThreads) hg[i] = hs[i];
}

__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t cluster_addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
  return v;
}

// Exclusive prefix sum over the block's 1024 threads (thread order).
__device__ __forceinline__ uint32_t block_scan_excl(uint32_t x, uint32_t* ws) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) ws[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t v = ws[lane];
    uint32_t vi = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, vi, o);
      if (lane >= o) vi += y;
    }
    ws[lane] = vi - v;
  }
  __syncthreads();
  const uint32_t r = ws[warp] + incl - x;
  __syncthreads();
  return r;
}

__device__ __forceinline__ uint64_t ld_cluster_u64(uint32_t cluster_addr) {
  uint64_t v;
  asm volatile("ld.shared::cluster.u64 %0, [%1];" : "=l"(v) : "r"(cluster_addr) : "memory");
  return v;
}

struct TopkShared {
  uint64_t list[kListCap];  // this CTA's candidates, ascending: key << 32 | position
  uint32_t keep_bits[kMaxWords], tie_bits[kMaxWords];
  int red[kPortion];        // this CTA's portion of the row's 12-bit histogram
  int hist1[1024], hist2[1024];
  uint32_t scan_ws[32];
  int warp_above[32], warp_inbin[32], warp_ibase[32];
  int seg_base[kClusterRanks + 1], seg_n[kClusterRanks], seg_above[kClusterRanks];
  int seg_gt[kClusterRanks], seg_tie[kClusterRanks];
  uint64_t bar;
  int abort_flag;
  int portion_total;
  int n_above, n_inbin;     // read by the peers (list mode)
  int owner, owner_above;
  int sel_bin, kk_new, bin_count;
  int n_keep, n_tie, cta_out, cta_tie_base, cta_keep;
};

constexpr int kTopkSharedBytes = round_up(static_cast<int>(sizeof(TopkShared)), 128);
static_assert(kTopkSharedBytes + kMaxSlice * 4 <= kSmemLimit && kMaxSlice * 4 >= kListCap * 8,
              "decode top-k shared memory");

// Each thread holds one bin (count c, index bin); thread order is descending
// bin order.  Records the bin that holds the kk-th largest key, given that
// `base_above` keys lie in bins above all of this block's bins.
__device__ __forceinline__ void pick_bin(int c, int bin, int kk, int base_above, TopkShared& sh) {
  const int above = base_above + static_cast<int>(block_scan_excl(static_cast<uint32_t>(c), sh.scan_ws));
  if (c > 0 && above < kk && above + c >= kk) {
    sh.sel_bin = bin;
    sh.kk_new = kk - above;
    sh.bin_count = c;
  }
  __syncthreads();
}

// Selection modes, chosen identically by every CTA of the cluster:
//   whole-bin  the 12-bit bin of the k-th key is taken entirely (or T <= k):
//              keep every key >= the bin's lower edge;
//   list       the bin holds at most kListCap keys in all: every CTA lists its
//              keys in the bin, gathers the whole cluster's lists and finishes
//              the selection locally (no further cluster barrier);
//   slice      a bin too full for the lists (heavy ties): two more 10-bit
//              passes over the slices with cluster-summed histograms.
__global__ void __cluster_dims__(kClusterRanks, 1, 1) __launch_bounds__(kTopkThreads, 1)
decode_topk_kernel(const uint32_t* __restrict__ keys, const int* __restrict__ hist, int n_split,
                   int32_t* __restrict__ idx, int row_stride, int T_max, const int* __restrict__ Ts, int k,
                   unsigned int* err) {
  extern __shared__ __align__(128) uint8_t topk_smem[];
  TopkShared& sh = *reinterpret_cast<TopkShared*>(topk_smem);
  uint32_t* slice = reinterpret_cast<uint32_t*>(topk_smem + kTopkSharedBytes);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned lt_mask = (1u << lane) - 1u;
  const int rank = static_cast<int>(cluster_ctarank());
  const size_t row = blockIdx.x / kClusterRanks;

  if (tid == 0) {
    mbar_init(&sh.bar, 1);
    sh.abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_trigger();
  pdl_wait();
  // the row's visible keys: one count for a uniform batch, per sequence when
  // varlen (uniform across the cluster: every CTA reads the same value)
  const int T = Ts ? min(max(__ldg(Ts + row), 0), T_max) : T_max;
  const int per = round_up((T + kClusterRanks - 1) / kClusterRanks, 4);
  const int lo = min(T, rank * per);
  const int n = min(T, lo + per) - lo;
  const int nw = (n + 31) / 32;
  if (tid == 0 && n > 0) {
    const uint32_t bytes = static_cast<uint32_t>(round_up(n, 4)) * 4u;
    mbar_arrive_expect_tx(&sh.bar, bytes);
    bulk_load_g2s(slice, keys + row * row_stride + lo, bytes, &sh.bar);
  }

  // ---- 12-bit bin of the k-th largest key, from the score kernel's
  // per-CTA histograms: CTA r sums bins [512 r, 512 r + 512) of the row
  const bool select = T > k;
  if (select && tid < kPortion) {
    const int* hrow = hist + row * n_split * kHistBins + rank * kPortion + tid;
    int part[4] = {0, 0, 0, 0};
    int s = 0;
    for (; s + 4 <= n_split; s += 4) {
#pragma unroll
      for (int u = 0; u < 4; ++u) part[u] += hrow[static_cast<size_t>(s + u) * kHistBins];
    }
    for (; s < n_split; ++s) part[0] += hrow[static_cast<size_t>(s) * kHistBins];
    sh.red[tid] = (part[0] + part[1]) + (part[2] + part[3]);
  }
  if (select) {
    const uint32_t part = tid < kPortion ? static_cast<uint32_t>(sh.red[tid]) : 0u;
    const uint32_t ex = block_scan_excl(part, sh.scan_ws);
    if (tid == kPortion - 1) sh.portion_total = static_cast<int>(ex + part);
  }
  cluster_sync();  // every portion is reduced

  uint32_t thr = 0u;   // keys >= thr (or > thr, when ties are limited) are kept
  int ties = 1 << 30;  // keys == thr granted, in position order
  uint32_t prefix = 0u;
  int kk = k;
  bool done = !select;
  bool list_mode = false;
  if (select) {
    if (warp == 0) {
      const int tot = lane < kClusterRanks
                          ? static_cast<int>(ld_cluster_u32(mapa_shared(smem_u32(&sh.portion_total), lane)))
                          : 0;
      int above = 0;
      for (int r = kClusterRanks - 1; r >= 0; --r) {
        const int tr = __shfl_sync(0xffffffffu, tot, r);
        if (above < k && above + tr >= k && lane == 0) {
          sh.owner = r;
          sh.owner_above = above;
        }
        above += tr;
      }
    }
    __syncthreads();
    const int owner = sh.owner;
    int c = 0;
    if (tid < kPortion)
      c = static_cast<int>(ld_cluster_u32(mapa_shared(smem_u32(&sh.red[kPortion - 1 - tid]), owner)));
    pick_bin(c, owner * kPortion + kPortion - 1 - tid, kk, sh.owner_above, sh);
    prefix = static_cast<uint32_t>(sh.sel_bin) << kHistShift;
    kk = sh.kk_new;
    if (sh.bin_count == kk) {  // the whole bin is taken
      thr = prefix;
      done = true;
    } else {
      list_mode = sh.bin_count <= kListCap;  // no CTA holds more than the bin's total
    }
  }
  if (n > 0 && !mbar_wait(&sh.bar, 0, &sh.abort_flag) && lane == 0) atomicOr(err, 1u);

  if (list_mode) {
    // ---- keys above the bin are kept; keys in it are listed in position
    // order (warp w owns a contiguous run of 32-key groups: count, scan, write)
    const uint32_t sel = prefix >> kHistShift;
    const int gpw = (nw + 31) / 32;
    const int g_lo = min(nw, warp * gpw), g_hi = min(nw, g_lo + gpw);
    int ca = 0, ci = 0;
    for (int g = g_lo; g < g_hi; ++g) {
      const int e = g * 32 + lane;
      const bool valid = e < n;
      const uint32_t top = (valid ? slice[e] : 0u) >> kHistShift;
      ca += __popc(__ballot_sync(0xffffffffu, valid && top > sel));
      ci += __popc(__ballot_sync(0xffffffffu, valid && top == sel));
    }
    if (lane == 0) { sh.warp_above[warp] = ca; sh.warp_inbin[warp] = ci; }
    __syncthreads();
    if (warp == 0) {
      const int a = sh.warp_above[lane], i = sh.warp_inbin[lane];
      int ai = a, ii = i;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int ya = __shfl_up_sync(0xffffffffu, ai, o), yi = __shfl_up_sync(0xffffffffu, ii, o);
        if (lane >= o) { ai += ya; ii += yi; }
      }
      sh.warp_ibase[lane] = ii - i;
      if (lane == 31) { sh.n_above = ai; sh.n_inbin = ii; }
    }
    __syncthreads();
    int base = sh.warp_ibase[warp];
    for (int g = g_lo; g < g_hi; ++g) {
      const int e = g * 32 + lane;
      const bool valid = e < n;
      const uint32_t key = valid ? slice[e] : 0u;
      const uint32_t top = key >> kHistShift;
      const unsigned above = __ballot_sync(0xffffffffu, valid && top > sel);
      const unsigned inbin = __ballot_sync(0xffffffffu, valid && top == sel);
      if (lane == 0) { sh.keep_bits[g] = above; sh.tie_bits[g] = 0u; }
      if ((inbin >> lane) & 1u)
        sh.list[base + __popc(inbin & lt_mask)] = (static_cast<uint64_t>(key) << 32) | static_cast<uint32_t>(lo + e);
      base += __popc(inbin);
    }
  }
  if (list_mode) cluster_sync();  // every CTA's list and counts are published

  if (list_mode) {
    // ---- gather the cluster's lists (ascending positions, rank by rank)
    // into the slice buffer, which list mode no longer needs
    uint64_t* all = reinterpret_cast<uint64_t*>(slice);
    if (warp == 0) {
      int ni = 0, na = 0;
      if (lane < kClusterRanks) {
        ni = static_cast<int>(ld_cluster_u32(mapa_shared(smem_u32(&sh.n_inbin), lane)));
        na = static_cast<int>(ld_cluster_u32(mapa_shared(smem_u32(&sh.n_above), lane)));
      }
      int incl = ni;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane < kClusterRanks) {
        sh.seg_base[lane] = incl - ni;
        sh.seg_n[lane] = ni;
        sh.seg_above[lane] = na;
        sh.seg_gt[lane] = 0;
        sh.seg_tie[lane] = 0;
      }
      if (lane == kClusterRanks - 1) sh.seg_base[kClusterRanks] = incl;
    }
    __syncthreads();
    const int m_all = sh.seg_base[kClusterRanks];
    const uint32_t list0 = smem_u32(&sh.list[0]);
    for (int i = tid; i < m_all; i += kTopkThreads) {
      int r = 0;
#pragma unroll
      for (int q = 1; q < kClusterRanks; ++q)
        if (i >= sh.seg_base[q]) r = q;
      all[i] = ld_cluster_u64(mapa_shared(list0 + 8u * static_cast<uint32_t>(i - sh.seg_base[r]), r));
    }
    cluster_arrive();  // this CTA reads no more peer memory
    __syncthreads();
    // ---- the remaining 20 bits of the k-th key, over the gathered list
    for (int pass = 0; pass < 2 && !done; ++pass) {
      const int shift = pass == 0 ? 10 : 0;
      const int hs = shift + 10;
      int* h = pass == 0 ? sh.hist1 : sh.hist2;
      h[tid] = 0;
      __syncthreads();
      for (int i = tid; i < m_all; i += kTopkThreads) {
        const uint32_t key = static_cast<uint32_t>(all[i] >> 32);
        if ((key >> hs) == (prefix >> hs)) atomicAdd(&h[(key >> shift) & 1023u], 1);
      }
      __syncthreads();
      pick_bin(h[1023 - tid], 1023 - tid, kk, 0, sh);
      prefix |= static_cast<uint32_t>(sh.sel_bin) << shift;
      kk = sh.kk_new;
      if (sh.bin_count == kk) done = true;  // the whole sub-bin is taken
    }
    thr = prefix;
    if (!done) ties = kk;
    const bool lim = ties < (1 << 30);
    // per-rank counts of kept and tied candidates; this CTA's own bits
    for (int i = tid; i < m_all; i += kTopkThreads) {
      int r = 0;
#pragma unroll
      for (int q = 1; q < kClusterRanks; ++q)
        if (i >= sh.seg_base[q]) r = q;
      const uint64_t ent = all[i];
      const uint32_t key = static_cast<uint32_t>(ent >> 32);
      const bool gt = lim ? key > thr : key >= thr;
      const bool tie = lim && key == thr;
      if (gt) atomicAdd(&sh.seg_gt[r], 1);
      if (tie) atomicAdd(&sh.seg_tie[r], 1);
      if (r == rank && (gt || tie)) {
        const int e = static_cast<int>(ent & 0xFFFFFFFFu) - lo;
        atomicOr(gt ? &sh.keep_bits[e >> 5] : &sh.tie_bits[e >> 5], 1u << (e & 31));
      }
    }
    __syncthreads();
    if (tid == 0) {
      int out_base = 0, tie_base = 0;
      for (int r = 0; r < rank; ++r) {
        out_base += sh.seg_above[r] + sh.seg_gt[r] + (lim ? max(0, min(sh.seg_tie[r], ties - tie_base)) : 0);
        tie_base += sh.seg_tie[r];
      }
      sh.cta_out = out_base;
      sh.cta_tie_base = tie_base;
    }
  } else {
    // ---- slice mode: two more radix passes over the slices
    if (!done) {
      for (int pass = 0; pass < 2 && !done; ++pass) {
        const int shift = pass == 0 ? 10 : 0;
        const int hs = shift + 10;
        int* h = pass == 0 ? sh.hist1 : sh.hist2;
        h[tid] = 0;
        __syncthreads();
        for (int e = tid; e < n; e += kTopkThreads) {
          const uint32_t key = slice[e];
          if ((key >> hs) == (prefix >> hs)) atomicAdd(&h[(key >> shift) & 1023u], 1);
        }
        cluster_sync();  // histograms of this pass complete (the two passes use separate buffers)
        int c = 0;
        const uint32_t a = smem_u32(&h[1023 - tid]);
#pragma unroll
        for (int r = 0; r < kClusterRanks; ++r) c += static_cast<int>(ld_cluster_u32(mapa_shared(a, r)));
        pick_bin(c, 1023 - tid, kk, 0, sh);
        prefix |= static_cast<uint32_t>(sh.sel_bin) << shift;
        kk = sh.kk_new;
        if (sh.bin_count == kk) done = true;  // the whole sub-bin is taken
      }
      thr = prefix;
      if (!done) ties = kk;  // thr is the exact k-th key; kk of its copies are taken
    }
    const bool lim = ties < (1 << 30);
    for (int g = warp; g < nw; g += kTopkThreads / 32) {
      const int e = g * 32 + lane;
      const bool valid = e < n;
      const uint32_t key = valid ? slice[e] : 0u;
      const unsigned kb = __ballot_sync(0xffffffffu, valid && (lim ? key > thr : key >= thr));
      const unsigned tb = __ballot_sync(0xffffffffu, valid && lim && key == thr);
      if (lane == 0) { sh.keep_bits[g] = kb; sh.tie_bits[g] = tb; }
    }
  }
  const bool limited = ties < (1 << 30);
  __syncthreads();

  // ---- ties in position order, then the output offsets.  Thread tid owns
  // bitmap words 2 tid and 2 tid + 1.
  const int w0 = 2 * tid;
  uint32_t kw[2] = {0u, 0u}, tw[2] = {0u, 0u};
#pragma unroll
  for (int j = 0; j < 2; ++j)
    if (w0 + j < nw) { kw[j] = sh.keep_bits[w0 + j]; tw[j] = sh.tie_bits[w0 + j]; }
  const uint32_t nk = __popc(kw[0]) + __popc(kw[1]), nt = __popc(tw[0]) + __popc(tw[1]);
  // keep and tie counts packed in one scan (each below 2^16 per CTA)
  const uint32_t ex = block_scan_excl((nk << 16) | nt, sh.scan_ws);
  if (!list_mode) {
    if (tid == kTopkThreads - 1) {
      sh.n_keep = static_cast<int>((ex >> 16) + nk);
      sh.n_tie = static_cast<int>((ex & 0xFFFFu) + nt);
    }
    cluster_sync();  // every CTA's totals are visible
    if (warp == 0) {
      int pk = 0, pt = 0;
      if (lane < rank) {
        pk = static_cast<int>(ld_cluster_u32(mapa_shared(smem_u32(&sh.n_keep), lane)));
        pt = static_cast<int>(ld_cluster_u32(mapa_shared(smem_u32(&sh.n_tie), lane)));
      }
      int out_base = 0, tie_base = 0;
      for (int r = 0; r < rank; ++r) {
        const int kr = __shfl_sync(0xffffffffu, pk, r), tr = __shfl_sync(0xffffffffu, pt, r);
        out_base += kr + (limited ? max(0, min(tr, ties - tie_base)) : 0);
        tie_base += tr;
      }
      if (lane == 0) { sh.cta_out = out_base; sh.cta_tie_base = tie_base; }
    }
    cluster_arrive();  // this CTA reads no more peer memory
  }
  __syncthreads();
  if (limited) {
    int tb = sh.cta_tie_base + static_cast<int>(ex & 0xFFFFu);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      uint32_t t = tw[j];
      int allowed = max(0, min(__popc(t), ties - tb));
      tb += __popc(t);
      while (allowed-- > 0) {
        kw[j] |= t & (0u - t);  // lowest remaining tied position
        t &= t - 1u;
      }
    }
  }
  const uint32_t mine = __popc(kw[0]) + __popc(kw[1]);
  const uint32_t off = block_scan_excl(mine, sh.scan_ws);
  if (tid == kTopkThreads - 1) sh.cta_keep = static_cast<int>(off + mine);
  int32_t* out = idx + row * k;
  int pos = sh.cta_out + static_cast<int>(off);
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    uint32_t bits = kw[j];
    while (bits) {
      const int bit = __ffs(bits) - 1;
      bits &= bits - 1u;
      if (pos < k) out[pos] = lo + (w0 + j) * 32 + bit;
      ++pos;
    }
  }
  __syncthreads();
  // padding when fewer than k positions are visible
  if (rank == kClusterRanks - 1) {
    for (int q = sh.cta_out + sh.cta_keep + tid; q < k; q += kTopkThreads) out[q] = -1;
  }
  cluster_wait();  // no CTA leaves while peers may read its shared memory
}

template <int H, int D>
dsa_status launch_dec(const CUtensorMap& tq, const CUtensorMap& tk, const DecParams& p, int grid,
                      cudaStream_t stream) {
  using C = DecCfg<H, D>;
  auto kern = decode_score_kernel<H, D>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), C::kSmem);
  if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("decode score smem attribute: ") + cudaGetErrorString(e));
  e = launch_pdl(kern, dim3(grid), dim3(kDecThreads), C::kSmem, stream, tq, tk, p);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("decode score launch: ") + cudaGetErrorString(e));
  return DSA_OK;
}

int score_splits(int B, int T, int sms) {
  const int tiles = (T + kTile - 1) / kTile;
  const int per_row = std::max(1, std::min(sms, kMaxScoreCtasPerRow) / B);
  return std::max(1, std::min(tiles, per_row));
}

size_t keys_bytes(int B, int Lk) {
  return (static_cast<size_t>(B) * round_up(Lk, 4) * 4 + 255) / 256 * 256;
}

}  // namespace

bool decode_indexer_applies(int Lq, int Lk, int start_pos, int H, int d) {
  const int T = start_pos;  // the single query row sits at t = start_pos
  return Lq == 1 && (H == 16 || H == 32 || H == 64) && (d == 64 || d == 128) && T >= 1 &&
         round_up((T + kClusterRanks - 1) / kClusterRanks, 4) <= kMaxSlice && Lk >= T;
}

size_t decode_indexer_ws_bytes(int B, int Lk) {
  // score keys, then per-CTA histograms for up to 160 score CTAs in all
  // (independent of the device's SM count)
  const size_t hist = static_cast<size_t>(B) * std::max(1, kMaxScoreCtasPerRow / B) * kHistBins * 4;
  return keys_bytes(B, Lk) + hist;
}

dsa_status decode_indexer_launch(const dsa_bf16* q_idx, const dsa_bf16* k_idx, const float* w, int B,
                                 int Lk, int start_pos, int H, int d, int k, int32_t* idx, void* ws,
                                 size_t ws_bytes, cudaStream_t stream, const DecodeVarlen* vl) {
  // uniform: every row at t = start_pos; varlen: row b at t = sp[b] <= Lk
  // (the batch's longest cache) over the packed keys
  const int T = vl ? Lk : start_pos;
  if (ws_bytes < decode_indexer_ws_bytes(B, Lk)) return set_error(DSA_ERR_WORKSPACE, "indexer workspace too small");
  const int sms = device_sm_count();
  if (sms <= 0) return set_error(DSA_ERR_CUDA, "cannot query the device SM count");
  const int n_split = score_splits(B, T, sms);
  const int tiles = (T + kTile - 1) / kTile;
  DecParams p{};
  p.w = w;
  p.keys = static_cast<uint32_t*>(ws);
  p.hist = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + keys_bytes(B, Lk));
  p.err = device_error_word();
  if (!p.err) return set_error(DSA_ERR_CUDA, "cannot resolve the device error word");
  p.sp = vl ? vl->sp : nullptr;
  p.cu_k = vl ? vl->cu_k : nullptr;
  p.B = B; p.row_stride = round_up(Lk, 4); p.T = T; p.n_split = n_split;
  p.split_len = ((tiles + n_split - 1) / n_split) * kTile;
  CUtensorMap tq, tk;
  if (!encode_tiled_3d(&tq, q_idx, d, H, B, static_cast<uint64_t>(d) * 2, static_cast<uint64_t>(H) * d * 2,
                       64, H, CU_TENSOR_MAP_SWIZZLE_128B))
    return set_error(DSA_ERR_CUDA, "tensor map for q_idx failed");
  const uint64_t krows = vl ? static_cast<uint64_t>(vl->total_k) : static_cast<uint64_t>(Lk);
  const uint64_t kbatch = vl ? 1u : static_cast<uint64_t>(B);
  if (!encode_tiled_3d(&tk, k_idx, d, krows, kbatch, static_cast<uint64_t>(d) * 2, krows * d * 2,
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
  const int per = round_up((T + kClusterRanks - 1) / kClusterRanks, 4);
  const int tsmem = kTopkSharedBytes + std::max(per * 4, kListCap * 8);
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(decode_topk_kernel), tsmem);
  if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("decode top-k smem attribute: ") + cudaGetErrorString(e));
  e = launch_pdl(decode_topk_kernel, dim3(B * kClusterRanks), dim3(kTopkThreads), tsmem, stream,
                 static_cast<const uint32_t*>(p.keys), static_cast<const int*>(p.hist), n_split, idx,
                 p.row_stride, T, p.sp, k, p.err);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("decode top-k launch: ") + cudaGetErrorString(e));
  return DSA_OK;
}

}  // namespace dsa
