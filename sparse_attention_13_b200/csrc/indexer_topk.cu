// indexer_topk.cu -- fused lightning indexer + streaming exact top-k (sm_100a).
//
// Computes, for every query row t, I[t,s] = sum_j w[t,j] ReLU(q[t,j].k[s]) over
// the visible keys s < t and keeps the k best positions ("注意力机制中的 Index",
// §4: index-score equation and TopK over s < t; ties go to the lower position,
// output ascending with -1 padding).  The L x L score matrix never exists.
//
// Design (one persistent CTA per SM, 320 threads):
//   warp 8   TMA producer: the 8-query block of q (resident, [8*H, d] bf16) and
//            a ring of 128-key tiles of k_idx, both 128B/64B-swizzled.
//   warp 9   UMMA issuer: per key tile and query half (4 queries) one
//            128 x (4H) x d MMA chain, D = keys x (query, head) in TMEM fp32,
//            double-buffered (2 x 256 columns).  Keys sit on the M side so each
//            TMEM lane is one key and the ReLU/head-weighted sum over the
//            4H columns of a query needs no cross-lane reduction.
//   warps 0-7 epilogue: tcgen05.ld a key's H head dots per query, fold
//            w[t,j]*max(dot,0) in fp32 (four chains over heads j mod 4 in a
//            fixed order, the same as the decode kernel's: deterministic),
//            pack (order-preserving score key << 32 | ~s) into one uint64 so a
//            plain integer order is (score desc, position asc), and append the
//            entries that beat the query's running threshold to a per-query
//            candidate buffer, in ascending s.  When a buffer passes 3k entries
//            an exact radix select (8-bit digits, in registers) keeps the best k
//            in place (stable) and raises the threshold to the k-th value.  At
//            the end of the block a final select writes the row.
// Few query blocks over long key ranges (short continuation chunks; single
// rows go to decode_indexer.cu where its shapes apply) split the key range
// across CTAs; each split keeps its own top-k and a merge kernel selects the
// final k.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstdio>

#include "dsa_internal.h"
#include "dsa_ptx.cuh"

namespace dsa {

namespace {

constexpr int kQB = 8;        // queries per work item
constexpr int kTileK = 128;   // keys per tile = UMMA M
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kThreads = (kEpiWarps + 2) * 32;
constexpr int kEpiBar = 1;
constexpr int kMaxK = 2048;
constexpr int kSelRows = (3 * kMaxK + kTileK + kEpiThreads - 1) / kEpiThreads;  // 25
constexpr int kMaxGrid = 160;
constexpr int kTmemCols = 512;
constexpr int kSmemBudget = 227 * 1024;

__host__ __device__ constexpr int cap_for(int k) { return 3 * k + kTileK; }

// Kernel shape.  bf16 operands: an MMA unit is one key tile against 4 queries
// (N = 4H, two units per tile).  MX operands (the low-precision selector of
// "注意力机制中的 Index" §5.4): 8-bit element codes, one K chunk of 128 bytes,
// units of 2 queries (N = 2H) so that the block scales fit in TMEM beside two
// accumulators.
template <int H, int D, bool MX = false>
struct Cfg {
  static constexpr int kElemBytes = MX ? 1 : 2;
  static constexpr int kChunkElems = MX ? D : (D < 64 ? D : 64);
  static constexpr int kChunkBytes = kChunkElems * kElemBytes;
  static constexpr int kChunks = D / kChunkElems;
  static constexpr uint32_t kSwz = kChunkBytes == 128 ? kSwizzle128B : kSwizzle64B;
  static constexpr int kSBO = 8 * kChunkBytes;
  static constexpr int kUnitQ = MX ? 2 : 4;                      // queries per MMA unit
  static constexpr int kUnits = kQB / kUnitQ;                    // units per key tile
  static constexpr int kQPT = kUnitQ / 2;                        // queries per epilogue thread in a unit
  static constexpr int kUnitRows = kUnitQ * H;                   // q rows of one unit (= N)
  static constexpr int kAccCols = kUnitRows;                     // TMEM columns of one accumulator
  static constexpr int kQUnitBytes = kUnitRows * kChunkBytes;    // one (chunk, unit) block
  static constexpr int kQBytes = kQB * H * D * kElemBytes;
  static constexpr int kKeyChunkBytes = kTileK * kChunkBytes;
  static constexpr int kStageBytes = kTileK * D * kElemBytes;
  static constexpr int kSfBytes = MX ? 512 : 0;                  // block scales of 128 rows
  static constexpr int kFixed = kQBytes + kUnits * kSfBytes + kQB * H * 4 + 8192;  // q + w + small state
  static constexpr int kStagesFit = (kSmemBudget - 1024 - kFixed) / (kStageBytes + kSfBytes);
  static constexpr int kMaxStages = MX ? 6 : 4;
  static constexpr int kStages = kStagesFit > kMaxStages ? kMaxStages : kStagesFit;
  // MX TMEM: accumulators [0, 2 kAccCols), key scales SFA[2] (4 columns each,
  // by tile parity), query scales SFB[2][kUnits] (4 columns each, by item parity)
  static constexpr uint32_t kSfaCol = 2 * kAccCols;
  static constexpr uint32_t kSfbCol = kSfaCol + 8;
  static_assert(kStages >= 2, "shared memory too small for two key stages");
  static_assert(kUnitRows <= 256, "TMA box rows");
  static_assert(kQUnitBytes % 512 == 0, "swizzle atom alignment");
  static_assert(!MX || (D == 128 && H == 64), "MX operands: d_I = 128, H_I = 64");
  static_assert(!MX || kSfbCol + 2 * kUnits * 4 <= kTmemCols, "MX TMEM layout");
  static_assert(MX || 2 * kAccCols <= kTmemCols, "TMEM accumulators");
};

struct SelShared {
  int hist[256];
  int wcnt[kSelRows][kEpiWarps];
  int woff[kSelRows][kEpiWarps];
  int sel_bin, kk_new, bin_count, total;
  uint32_t wlo[kEpiWarps], whi[kEpiWarps];  // per-warp key range
  unsigned long long minval;
};

struct EpiShared {
  unsigned long long thr[kQB];
  int lim[kQB];         // per query slot: keys s < lim are candidates (0: no query row)
  int cnt[2][kQB];
  int qcount[2][kQB][4];
  SelShared sel;
};

struct Params {
  const float* w;        // [rows, H]
  int32_t* idx;          // [rows, k]
  uint64_t* cand;        // [grid][kQB][cap]
  uint64_t* split_out;   // [rows][S][k]
  int* split_cnt;        // [rows][S]
  unsigned int* err;     // device error word
  // Variable-length batches (all three null for a uniform batch): sequence
  // b's query rows are cu_q[b] .. cu_q[b+1]-1 of the packed tensors, its keys
  // rows cu_k[b] .. cu_k[b+1]-1, and its first query row sits at sp[b].
  const int* cu_q;
  const int* cu_k;
  const int* sp;
  int B, Lq, Lk, start_pos, k, cap;  // Lq, Lk: the maxima over the batch when varlen
  int S, split_len, n_qblocks, n_items;
  // MX operands (uniform batches): block scales in the TMEM-copy layout, 512
  // bytes per group of 128 rows (query rows of one batch: [sfq_groups], key
  // rows: [sfk_tiles]); the block-scaled instruction descriptor without N.
  const uint8_t* sfq;
  const uint8_t* sfk;
  int sfq_groups, sfk_tiles;
  uint32_t mx_idesc;
};

struct Item {
  int b, qb, split;
  int s_begin, s_end;   // key range [s_begin, s_end) scanned by this item
  int n_tiles;
  int nvalid;           // valid queries of the block (may be <= 0 past the sequence)
  int lq, start;        // the sequence's query rows and its first row's position
  int q_row0, k_row0;   // first query / key row of the sequence in the q / k tensor maps
  int tb;               // batch coordinate of the tensor maps
  size_t out_row0;      // row of the sequence's first query in w, idx and the split lists
};

// valid queries of MMA unit u (unitq queries per unit)
__device__ __forceinline__ int unit_queries(const Item& it, int u, int unitq) {
  return max(0, min(unitq, it.nvalid - unitq * u));
}

__device__ __forceinline__ Item decode_item(const Params& p, int w) {
  Item it;
  it.split = w % p.S;
  const int rest = w / p.S;
  it.b = rest % p.B;
  it.qb = p.n_qblocks - 1 - rest / p.B;  // longest query blocks first
  if (p.cu_q) {
    const int q0 = __ldg(p.cu_q + it.b);
    it.lq = min(max(__ldg(p.cu_q + it.b + 1) - q0, 0), p.Lq);
    it.start = max(__ldg(p.sp + it.b), 0);
    it.q_row0 = q0;
    it.k_row0 = __ldg(p.cu_k + it.b);
    it.tb = 0;
    it.out_row0 = static_cast<size_t>(q0);
  } else {
    it.lq = p.Lq;
    it.start = p.start_pos;
    it.q_row0 = 0;
    it.k_row0 = 0;
    it.tb = it.b;
    it.out_row0 = static_cast<size_t>(it.b) * p.Lq;
  }
  const int i0 = it.qb * kQB;
  const int nvalid = min(kQB, it.lq - i0);
  it.nvalid = nvalid;
  const int t_max = it.start + i0 + nvalid - 1;  // largest visible count in the block
  it.s_begin = it.split * p.split_len;
  it.s_end = min(t_max, it.s_begin + p.split_len);
  it.n_tiles = nvalid > 0 && it.s_end > it.s_begin ? (it.s_end - it.s_begin + kTileK - 1) / kTileK : 0;
  return it;
}

// Item sequence of a CTA: snake order over rounds of `grid` items.
__device__ __forceinline__ int item_of(int round, int cta, int grid) {
  return round * grid + ((round & 1) ? (grid - 1 - cta) : cta);
}

__device__ __forceinline__ unsigned long long pack_entry(float score, int s) {
  return (static_cast<unsigned long long>(float_key(score)) << 32) |
         static_cast<unsigned long long>(~static_cast<uint32_t>(s));
}

// ------------------------------------------------------------------ select
// Exclusive prefix of per-(row, warp) counts over the 256 epilogue threads in
// (row, warp, lane) order; writes sh.woff and returns the total.
__device__ __forceinline__ int scan_rows(const unsigned (&mask)[kSelRows], SelShared& sh) {
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
#pragma unroll
  for (int r = 0; r < kSelRows; ++r)
    if (lane == 0) sh.wcnt[r][warp] = __popc(mask[r]);
  named_bar_sync(kEpiBar, kEpiThreads);
  if (warp == 0) {
    constexpr int kN = kSelRows * kEpiWarps;
    constexpr int kPer = (kN + 31) / 32;
    int loc[kPer];
    int sum = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = lane * kPer + i;
      loc[i] = e < kN ? (&sh.wcnt[0][0])[e] : 0;
      sum += loc[i];
    }
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    int run = incl - sum;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = lane * kPer + i;
      if (e < kN) (&sh.woff[0][0])[e] = run;
      run += loc[i];
    }
    if (lane == 31) sh.total = incl;
  }
  named_bar_sync(kEpiBar, kEpiThreads);
  return sh.total;
}

// Exact top-k of buf[0, cnt): distinct uint64 entries (score key << 32 | ~s)
// held in ascending-position order, by all 256 epilogue threads.  The radix
// select runs on the 32-bit score key only; entries tied with the threshold
// key are taken in buffer order, i.e. lowest position first, which is the
// (score desc, position asc) order.  mode 0: keep the best k in place
// (stable) and return the smallest kept entry.  mode 1: write the selected
// positions to out_idx (ascending) and pad with -1 up to k.  mode 2: copy the
// selected entries to out_list and their number to *out_count.
__device__ unsigned long long select_topk(const uint64_t* src, uint64_t* dst_inplace,
                                          int cnt, int k, int mode, int32_t* out_idx,
                                          uint64_t* out_list, int* out_count, SelShared& sh) {
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const unsigned lt = (1u << lane) - 1u;
  unsigned long long v[kSelRows];
#pragma unroll
  for (int r = 0; r < kSelRows; ++r) {
    const int e = r * kEpiThreads + tid;
    v[r] = e < cnt ? src[e] : 0ull;
  }
  uint32_t thr = 0u;       // threshold score key
  int ties = 1 << 30;      // how many entries equal to thr are kept (in order)
  if (cnt > k) {
    // The bits above the highest one in which the smallest and the largest key
    // differ are common to all entries, so the radix starts at that bit: the
    // first digit spreads the entries over the bins instead of piling them into
    // the one or two bins of a shared exponent, and the passes over common
    // bits are skipped.
    uint32_t lo = ~0u, hi = 0u;
#pragma unroll
    for (int r = 0; r < kSelRows; ++r) {
      const uint32_t key = static_cast<uint32_t>(v[r] >> 32);
      if (r * kEpiThreads + tid < cnt) {
        lo = key < lo ? key : lo;
        hi = key > hi ? key : hi;
      }
    }
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    if (lane == 0) { sh.wlo[warp] = lo; sh.whi[warp] = hi; }
    named_bar_sync(kEpiBar, kEpiThreads);
#pragma unroll
    for (int w = 0; w < kEpiWarps; ++w) {
      lo = sh.wlo[w] < lo ? sh.wlo[w] : lo;
      hi = sh.whi[w] > hi ? sh.whi[w] : hi;
    }
    const uint32_t diff = lo ^ hi;
    const int hb = diff ? 31 - __clz(diff) : -1;   // highest differing bit
    uint32_t prefix = hb < 0 ? hi : hi & ~((2u << hb) - 1u);  // hb = 31: 2u << 31 wraps to 0
    int kk = k;
    bool exact = true;     // the loop ran down to a single key value
    for (int shift = hb - 7; hb >= 0;) {
      int width = 8;
      if (shift < 0) { width += shift; shift = 0; }
      const int top = shift + width;               // bits >= top are fixed by prefix
      const uint32_t dmask = (1u << width) - 1u;
      if (tid < 256) sh.hist[tid] = 0;
      named_bar_sync(kEpiBar, kEpiThreads);
#pragma unroll
      for (int r = 0; r < kSelRows; ++r) {
        const int e = r * kEpiThreads + tid;
        if (e < cnt) {
          const uint32_t key = static_cast<uint32_t>(v[r] >> 32);
          if (top == 32 || (key >> top) == (prefix >> top))
            atomicAdd(&sh.hist[(key >> shift) & dmask], 1);
        }
      }
      named_bar_sync(kEpiBar, kEpiThreads);
      if (warp == 0) {
        int loc[8];
        int sum = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) { loc[i] = sh.hist[lane * 8 + i]; sum += loc[i]; }
        int incl = sum;  // inclusive suffix sum over lanes >= lane
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int y = __shfl_down_sync(0xffffffffu, incl, off);
          if (lane + off < 32) incl += y;
        }
        int above = incl - sum;  // entries in bins of higher lanes
#pragma unroll
        for (int i = 7; i >= 0; --i) {
          if (above < kk && above + loc[i] >= kk) {
            sh.sel_bin = lane * 8 + i;
            sh.kk_new = kk - above;
            sh.bin_count = loc[i];
          }
          above += loc[i];
        }
      }
      named_bar_sync(kEpiBar, kEpiThreads);
      prefix |= static_cast<uint32_t>(sh.sel_bin) << shift;
      kk = sh.kk_new;
      if (sh.bin_count == kk) {  // the whole bin is selected: keep every key >= prefix
        exact = false;
        break;
      }
      if (shift == 0) break;
      shift -= 8;
    }
    thr = prefix;          // hb < 0: every key equals hi, the first k are kept
    if (exact) ties = kk;
  }
  // keep decision: key > thr, or key == thr within the first `ties` such entries
  bool keep[kSelRows];
  unsigned mask[kSelRows];
  bool limited = ties < (1 << 30);
#pragma unroll
  for (int r = 0; r < kSelRows; ++r) {
    const int e = r * kEpiThreads + tid;
    const uint32_t key = static_cast<uint32_t>(v[r] >> 32);
    keep[r] = e < cnt && (limited ? key > thr : key >= thr);
    mask[r] = __ballot_sync(0xffffffffu, e < cnt && limited && key == thr);
  }
  if (limited) {
    scan_rows(mask, sh);
#pragma unroll
    for (int r = 0; r < kSelRows; ++r)
      if (mask[r] & (1u << lane))
        keep[r] = keep[r] || (sh.woff[r][warp] + __popc(mask[r] & lt) < ties);
    named_bar_sync(kEpiBar, kEpiThreads);  // woff is reused below
  }
#pragma unroll
  for (int r = 0; r < kSelRows; ++r) mask[r] = __ballot_sync(0xffffffffu, keep[r]);
  if (tid == 0) sh.minval = ~0ull;
  const int total = scan_rows(mask, sh);
  unsigned long long local_min = ~0ull;
#pragma unroll
  for (int r = 0; r < kSelRows; ++r) {
    if (keep[r]) {
      const int pos = sh.woff[r][warp] + __popc(mask[r] & lt);
      if (mode == 0) {
        dst_inplace[pos] = v[r];
        local_min = v[r] < local_min ? v[r] : local_min;
      } else if (mode == 1) {
        out_idx[pos] = static_cast<int32_t>(~static_cast<uint32_t>(v[r] & 0xffffffffull));
      } else {
        out_list[pos] = v[r];
      }
    }
  }
  unsigned long long result = 0ull;
  if (mode == 0) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const unsigned long long o = __shfl_xor_sync(0xffffffffu, local_min, off);
      local_min = o < local_min ? o : local_min;
    }
    if (lane == 0) atomicMin(&sh.minval, local_min);
    named_bar_sync(kEpiBar, kEpiThreads);
    result = sh.minval;
  } else if (mode == 1) {
    for (int pos = total + tid; pos < k; pos += kEpiThreads) out_idx[pos] = -1;
  } else {
    if (tid == 0) *out_count = total;
  }
  named_bar_sync(kEpiBar, kEpiThreads);
  return result;
}

// ------------------------------------------------------------------ kernel
template <int H, int D, bool MX>
__global__ void __launch_bounds__(kThreads, 1)
indexer_topk_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k, const Params p) {
  using C = Cfg<H, D, MX>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* q_smem = smem;
  uint8_t* key_smem = q_smem + C::kQBytes;
  // MX: the query block's scales (kUnits x 512 B), then one 512 B block per key stage
  uint8_t* sfq_smem = key_smem + C::kStages * C::kStageBytes;
  uint8_t* sfk_smem = sfq_smem + C::kUnits * C::kSfBytes;
  float* w_smem = reinterpret_cast<float*>(sfk_smem + C::kStages * C::kSfBytes);
  EpiShared* es = reinterpret_cast<EpiShared*>(w_smem + kQB * H);
  uint64_t* bars = reinterpret_cast<uint64_t*>(es + 1);
  uint64_t* key_full = bars;
  uint64_t* key_empty = bars + C::kStages;
  uint64_t* tmem_full = bars + 2 * C::kStages;
  uint64_t* tmem_empty = tmem_full + 2;
  uint64_t* q_full = tmem_empty + 2;
  uint64_t* q_empty = q_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* consumed_tiles = abort_flag + 1;  // key tiles retired by the MMA warp

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const int grid = gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) { mbar_init(&key_full[s], 1); mbar_init(&key_empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&tmem_full[b], 1); mbar_init(&tmem_empty[b], kEpiWarps); }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    *abort_flag = 0;
    *consumed_tiles = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kTmaWarp && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_trigger();
  pdl_wait();

  int issued_tiles = 0;  // producer lane 0 only
  if (warp == kTmaWarp) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int n_items_done = 0;
      for (int round = 0;; ++round) {
        const int w = item_of(round, cta, grid);
        if (round * grid >= p.n_items) break;
        if (w >= p.n_items) continue;
        const Item it = decode_item(p, w);
        if (it.n_tiles == 0) continue;
        if (!mbar_wait(q_empty, (n_items_done & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(q_full, C::kQBytes + C::kUnits * C::kSfBytes);
        for (int c = 0; c < C::kChunks; ++c)
          for (int h = 0; h < C::kUnits; ++h)
            tma_load_3d(q_smem + (c * C::kUnits + h) * C::kQUnitBytes, &tm_q, q_full,
                        c * C::kChunkElems, (it.q_row0 + it.qb * kQB + C::kUnitQ * h) * H, it.tb);
        if constexpr (MX)  // the block's kUnits scale groups are contiguous
          bulk_load_g2s(sfq_smem, p.sfq + (static_cast<size_t>(it.tb) * p.sfq_groups + it.qb * C::kUnits) * 512,
                        C::kUnits * C::kSfBytes, q_full);
        bool ok = true;
        for (int j = 0; j < it.n_tiles; ++j) {
          if (!mbar_wait(&key_empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&key_full[stage], C::kStageBytes + C::kSfBytes);
          uint8_t* dst = key_smem + stage * C::kStageBytes;
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_3d(dst + c * C::kKeyChunkBytes, &tm_k, &key_full[stage],
                        c * C::kChunkElems, it.k_row0 + it.s_begin + j * kTileK, it.tb);
          if constexpr (MX)
            bulk_load_g2s(sfk_smem + stage * C::kSfBytes,
                          p.sfk + (static_cast<size_t>(it.tb) * p.sfk_tiles + (it.s_begin + j * kTileK) / kTileK) * 512,
                          C::kSfBytes, &key_full[stage]);
          ++issued_tiles;
          if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        ++n_items_done;
      }
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------- UMMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t unit = 0;
      int n_items_done = 0;
      bool ok = true;
      for (int round = 0; ok; ++round) {
        const int w = item_of(round, cta, grid);
        if (round * grid >= p.n_items) break;
        if (w >= p.n_items) continue;
        const Item it = decode_item(p, w);
        if (it.n_tiles == 0) continue;
        if (!mbar_wait(q_full, n_items_done & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t sfb_col = C::kSfbCol + (n_items_done & 1) * C::kUnits * 4;
        if constexpr (MX) {
          // the query block's scales into TMEM (this item's parity): tcgen05
          // copies and MMAs of one thread run in issue order
          for (int h = 0; h < C::kUnits; ++h)
            tc_cp_32x128b_x4(tmem_base + sfb_col + 4 * h,
                             make_smem_desc(smem_u32(sfq_smem + h * C::kSfBytes), 16, 128, kSwizzleNone));
        }
        for (int j = 0; j < it.n_tiles && ok; ++j) {
          if (!mbar_wait(&key_full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(key_smem + stage * C::kStageBytes);
          const uint32_t sfa_col = C::kSfaCol + (*consumed_tiles & 1) * 4;
          if constexpr (MX)
            tc_cp_32x128b_x4(tmem_base + sfa_col,
                             make_smem_desc(smem_u32(sfk_smem + stage * C::kSfBytes), 16, 128, kSwizzleNone));
          for (int h = 0; h < C::kUnits; ++h) {
            if (unit_queries(it, h, C::kUnitQ) == 0) continue;
            const uint32_t buf = unit & 1;
            if (!mbar_wait(&tmem_empty[buf], ((unit >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const int n = ((unit_queries(it, h, C::kUnitQ) * H + 15) / 16) * 16;
            const uint32_t d_tmem = tmem_base + buf * C::kAccCols;
            const uint32_t b_base = smem_u32(q_smem) + h * C::kQUnitBytes;
            if constexpr (MX) {
              // four K = 32 steps; step kk takes byte kk of the scale columns
              const uint32_t idesc = p.mx_idesc | (static_cast<uint32_t>(n >> 3) << 17);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = make_smem_desc(a_base + kk * 32, 16, C::kSBO, C::kSwz);
                const uint64_t bd = make_smem_desc(b_base + kk * 32, 16, C::kSBO, C::kSwz);
                umma_mx_ss(d_tmem, ad, bd, idesc | mx_sf_ids(kk, kk), tmem_base + sfa_col,
                           tmem_base + sfb_col + 4 * h, kk != 0);
              }
            } else {
              const uint32_t idesc = make_idesc_bf16(128, n, 0, 0);
#pragma unroll
              for (int c = 0; c < C::kChunks; ++c) {
#pragma unroll
                for (int kk = 0; kk < C::kChunkElems / 16; ++kk) {
                  const uint64_t ad = make_smem_desc(a_base + c * C::kKeyChunkBytes + kk * 32, 16,
                                                     C::kSBO, C::kSwz);
                  const uint64_t bd = make_smem_desc(b_base + c * C::kUnits * C::kQUnitBytes + kk * 32, 16,
                                                     C::kSBO, C::kSwz);
                  umma_bf16_ss(d_tmem, ad, bd, idesc, (c | kk) != 0);
                }
              }
            }
            umma_commit(&tmem_full[buf]);
            ++unit;
          }
          umma_commit(&key_empty[stage]);
          *consumed_tiles = *consumed_tiles + 1;
          if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        }
        umma_commit(q_empty);
        ++n_items_done;
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const int qd = warp & 3;       // TMEM lane quadrant
    const int qg = warp >> 2;      // query group within a half (kQPT queries)
    const int tid = threadIdx.x;
    uint32_t unit = 0;
    for (int round = 0;; ++round) {
      const int w = item_of(round, cta, grid);
      if (round * grid >= p.n_items) break;
      if (w >= p.n_items) continue;
      const Item it = decode_item(p, w);
      const int i0 = it.qb * kQB;
      // per-item state
      if (tid < kQB) {
        es->thr[tid] = 0ull;
        es->cnt[0][tid] = 0;
        // row i0 + tid sees s < t = start + i0 + tid, within this item's key range
        es->lim[tid] = i0 + tid < it.lq ? min(it.start + i0 + tid, it.s_end) : 0;
      }
      for (int e = tid; e < kQB * H; e += kEpiThreads) {
        const int qs = e / H;
        const int i = i0 + qs;
        w_smem[e] = i < it.lq ? p.w[(it.out_row0 + i) * H + (e % H)] : 0.f;
      }
      named_bar_sync(kEpiBar, kEpiThreads);
      uint64_t* cand_base = p.cand + static_cast<size_t>(cta) * kQB * p.cap;
      bool ok = true;
      for (int j = 0; j < it.n_tiles && ok; ++j) {
        const int par = j & 1;
        const int s = it.s_begin + j * kTileK + qd * 32 + lane;
        for (int h = 0; h < C::kUnits; ++h) {
          if (unit_queries(it, h, C::kUnitQ) == 0) continue;
          const uint32_t buf = unit & 1;
          if (!__all_sync(0xffffffffu, mbar_wait(&tmem_full[buf], (unit >> 1) & 1, abort_flag))) { ok = false; break; }
          tc_fence_after();
          float acc[C::kQPT];
          const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(qd * 32) << 16) + buf * C::kAccCols;
          if constexpr (H >= 32) {
            uint32_t v[C::kQPT][H];
#pragma unroll
            for (int jj = 0; jj < C::kQPT; ++jj)
#pragma unroll
              for (int c = 0; c < H / 32; ++c)
                tmem_ld32<32>(t_lane + (C::kQPT * qg + jj) * H + c * 32,
                              *reinterpret_cast<uint32_t(*)[32]>(&v[jj][c * 32]));
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tmem_empty[buf]);
            // heads j = 4c + r accumulate into a[r] (four independent FMA
            // chains), combined as (a0 + a1) + (a2 + a3)
#pragma unroll
            for (int jj = 0; jj < C::kQPT; ++jj) {
              const float4* w4 = reinterpret_cast<const float4*>(w_smem + (C::kUnitQ * h + C::kQPT * qg + jj) * H);
              float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
              for (int c = 0; c < H / 4; ++c) {
                const float4 ww = w4[c];
                a[0] = fmaf(fmaxf(__uint_as_float(v[jj][4 * c + 0]), 0.f), ww.x, a[0]);
                a[1] = fmaf(fmaxf(__uint_as_float(v[jj][4 * c + 1]), 0.f), ww.y, a[1]);
                a[2] = fmaf(fmaxf(__uint_as_float(v[jj][4 * c + 2]), 0.f), ww.z, a[2]);
                a[3] = fmaf(fmaxf(__uint_as_float(v[jj][4 * c + 3]), 0.f), ww.w, a[3]);
              }
              acc[jj] = (a[0] + a[1]) + (a[2] + a[3]);
            }
          } else {
            uint32_t v[C::kQPT][H];
#pragma unroll
            for (int jj = 0; jj < C::kQPT; ++jj)
              tmem_ld32<H>(t_lane + (C::kQPT * qg + jj) * H, v[jj]);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tmem_empty[buf]);
#pragma unroll
            for (int jj = 0; jj < C::kQPT; ++jj) {
              const float* wq = w_smem + (C::kUnitQ * h + C::kQPT * qg + jj) * H;
              float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
              for (int c = 0; c < H; ++c) a[c & 3] = fmaf(fmaxf(__uint_as_float(v[jj][c]), 0.f), wq[c], a[c & 3]);
              acc[jj] = (a[0] + a[1]) + (a[2] + a[3]);
            }
          }
          if constexpr (MX) {
            // the low-precision selector ranks scores quantised from fp32 to
            // bf16 (round to nearest even)
#pragma unroll
            for (int jj = 0; jj < C::kQPT; ++jj) acc[jj] = __bfloat162float(__float2bfloat16_rn(acc[jj]));
          }
          // candidate test and ordered append
          unsigned long long P[C::kQPT];
          unsigned msk[C::kQPT];
#pragma unroll
          for (int jj = 0; jj < C::kQPT; ++jj) {
            const int qs = C::kUnitQ * h + C::kQPT * qg + jj;
            const bool valid = s < es->lim[qs];
            P[jj] = pack_entry(acc[jj], s);
            const bool cand = valid && P[jj] > es->thr[qs];
            msk[jj] = __ballot_sync(0xffffffffu, cand);
            if (lane == 0) es->qcount[par][qs][qd] = __popc(msk[jj]);
          }
          named_bar_sync(kEpiBar, kEpiThreads);
          bool need_sel = false;
#pragma unroll
          for (int jj = 0; jj < C::kQPT; ++jj) {
            const int qs = C::kUnitQ * h + C::kQPT * qg + jj;
            const int base = es->cnt[par][qs];
            int off = base;
            for (int x = 0; x < qd; ++x) off += es->qcount[par][qs][x];
            if (msk[jj] & (1u << lane)) {
              cand_base[static_cast<size_t>(qs) * p.cap + off + __popc(msk[jj] & ((1u << lane) - 1u))] = P[jj];
            }
          }
          // every thread derives the new counts of the unit's queries
          int newcnt[C::kUnitQ];
#pragma unroll
          for (int q4 = 0; q4 < C::kUnitQ; ++q4) {
            const int qs = C::kUnitQ * h + q4;
            newcnt[q4] = es->cnt[par][qs] + es->qcount[par][qs][0] + es->qcount[par][qs][1] +
                         es->qcount[par][qs][2] + es->qcount[par][qs][3];
            need_sel |= newcnt[q4] > p.cap - kTileK;
          }
          if (tid < C::kUnitQ) es->cnt[par ^ 1][C::kUnitQ * h + tid] = newcnt[tid];
          if (need_sel) {
            named_bar_sync(kEpiBar, kEpiThreads);  // appends and counts visible
#pragma unroll 1
            for (int q4 = 0; q4 < C::kUnitQ; ++q4) {
              if (newcnt[q4] <= p.cap - kTileK) continue;
              const int qs = C::kUnitQ * h + q4;
              uint64_t* bq = cand_base + static_cast<size_t>(qs) * p.cap;
              const unsigned long long kth =
                  select_topk(bq, bq, newcnt[q4], p.k, 0, nullptr, nullptr, nullptr, es->sel);
              if (tid == 0) {
                es->thr[qs] = kth;
                es->cnt[par ^ 1][qs] = p.k;
              }
            }
            named_bar_sync(kEpiBar, kEpiThreads);
          }
          ++unit;
        }
      }
      if (!ok) break;
      // final selection per query row (the item's placement is decoded again
      // here rather than kept in registers through the tile loop)
      named_bar_sync(kEpiBar, kEpiThreads);
      const int fpar = it.n_tiles & 1;
      const Item itf = decode_item(p, w);
#pragma unroll 1
      for (int qs = 0; qs < kQB; ++qs) {
        const int i = i0 + qs;
        if (i >= itf.lq) break;
        const int c = es->cnt[fpar][qs];
        const uint64_t* bq = cand_base + static_cast<size_t>(qs) * p.cap;
        const size_t row = itf.out_row0 + i;
        if (p.S == 1) {
          select_topk(bq, nullptr, c, p.k, 1, p.idx + row * p.k, nullptr, nullptr, es->sel);
        } else {
          const size_t slot = row * p.S + itf.split;
          select_topk(bq, nullptr, c, p.k, 2, nullptr, p.split_out + slot * p.k,
                      p.split_cnt + slot, es->sel);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && warp == kTmaWarp && lane == 0) {
    // Abort path only: let key-tile loads that no MMA consumed land before
    // the CTA's shared memory is released (bounded; a load that never lands
    // leaves nothing more to do).
    for (int t = *consumed_tiles; t < issued_tiles; ++t) {
      const uint32_t a = smem_u32(&key_full[t % C::kStages]);
      const uint32_t par = (t / C::kStages) & 1;
      const long long t0 = clock64();
      while (!mbar_try_wait(a, par) && clock64() - t0 < kWaitLimitCycles) {}
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) atomicOr(p.err, 1u);
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ------------------------------------------------------------------ merge
// Final top-k over the S per-split candidate lists of one query row.  The
// lists concatenated in split order are in ascending position order, so the
// 32-bit score keys are radix-selected in shared memory and ties at the
// threshold are taken in that order; a stable compaction writes the row.
constexpr int kMergeThreads = 1024;
constexpr int kMaxSplits = 16;

__device__ __forceinline__ int block_excl_scan(int x, int* warp_sums, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int w = warp_sums[lane];
    int wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += y;
    }
    warp_sums[lane] = wi - w;
    if (lane == 31) warp_sums[32] = wi;
  }
  __syncthreads();
  const int r = warp_sums[warp] + incl - x;
  total = warp_sums[32];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kMergeThreads)
indexer_merge_kernel(const uint64_t* __restrict__ split_out, const int* __restrict__ split_cnt,
                     int32_t* __restrict__ idx, int S, int k) {
  extern __shared__ uint32_t keys[];  // [S * k] score keys in union order
  __shared__ int off[kMaxSplits + 1];
  __shared__ int hist[256];
  __shared__ int warp_sums[33];
  __shared__ int sel_bin, kk_new, bin_count;
  pdl_trigger();
  pdl_wait();
  const size_t row = blockIdx.x;
  const int tid = threadIdx.x;
  const uint64_t* lists = split_out + row * S * k;
  if (tid == 0) {
    int acc = 0;
    for (int j = 0; j < S; ++j) { off[j] = acc; acc += split_cnt[row * S + j]; }
    off[S] = acc;
  }
  __syncthreads();
  const int n = off[S];
  {
    int j = 0;
    for (int e = tid; e < n; e += kMergeThreads) {
      while (off[j + 1] <= e) ++j;
      keys[e] = static_cast<uint32_t>(lists[static_cast<size_t>(j) * k + (e - off[j])] >> 32);
    }
  }
  __syncthreads();
  uint32_t thr = 0u;
  int ties = 1 << 30;
  if (n > k) {
    uint32_t prefix = 0u;
    int kk = k;
    bool exact = true;
    for (int shift = 24; shift >= 0; shift -= 8) {
      if (tid < 256) hist[tid] = 0;
      __syncthreads();
      for (int e = tid; e < n; e += kMergeThreads) {
        const uint32_t key = keys[e];
        if (shift == 24 || (key >> (shift + 8)) == (prefix >> (shift + 8)))
          atomicAdd(&hist[(key >> shift) & 255u], 1);
      }
      __syncthreads();
      if (tid < 32) {
        int loc[8];
        int sum = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) { loc[i] = hist[tid * 8 + i]; sum += loc[i]; }
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
            sel_bin = tid * 8 + i;
            kk_new = kk - above;
            bin_count = loc[i];
          }
          above += loc[i];
        }
      }
      __syncthreads();
      prefix |= static_cast<uint32_t>(sel_bin) << shift;
      kk = kk_new;
      const bool whole_bin = bin_count == kk;
      __syncthreads();
      if (whole_bin) {
        exact = false;
        break;
      }
    }
    thr = prefix;
    if (exact) ties = kk;
  }
  const bool limited = ties < (1 << 30);
  // stable compaction over contiguous segments of the union
  const int per = (n + kMergeThreads - 1) / kMergeThreads;
  const int e0 = min(n, tid * per), e1 = min(n, e0 + per);
  int n_tie = 0;
  if (limited)
    for (int e = e0; e < e1; ++e) n_tie += keys[e] == thr;
  int tie_total;
  int tie_rank = block_excl_scan(n_tie, warp_sums, tie_total);
  int n_keep = 0;
  {
    int tr = tie_rank;
    for (int e = e0; e < e1; ++e) {
      const uint32_t key = keys[e];
      bool kp;
      if (limited) {
        kp = key > thr || (key == thr && tr < ties);
        tr += key == thr;
      } else {
        kp = key >= thr;
      }
      n_keep += kp;
    }
  }
  int total;
  int pos = block_excl_scan(n_keep, warp_sums, total);
  int32_t* out = idx + row * k;
  {
    int tr = tie_rank;
    int j = 0;
    for (int e = e0; e < e1; ++e) {
      const uint32_t key = keys[e];
      bool kp;
      if (limited) {
        kp = key > thr || (key == thr && tr < ties);
        tr += key == thr;
      } else {
        kp = key >= thr;
      }
      if (kp) {
        while (off[j + 1] <= e) ++j;
        const uint64_t v = lists[static_cast<size_t>(j) * k + (e - off[j])];
        out[pos++] = static_cast<int32_t>(~static_cast<uint32_t>(v & 0xffffffffull));
      }
    }
  }
  for (int q = total + tid; q < k; q += kMergeThreads) out[q] = -1;
}

template <int H, int D, bool MX = false>
dsa_status launch_hd(const CUtensorMap& tq, const CUtensorMap& tk, const Params& p, int grid,
                     cudaStream_t stream) {
  using C = Cfg<H, D, MX>;
  // At least 120 KB so that one CTA owns each SM (and all of its TMEM).
  const int smem = std::max(120 * 1024, 1024 + C::kQBytes + C::kStages * C::kStageBytes +
                                            (C::kUnits + C::kStages) * C::kSfBytes +
                                            kQB * H * 4 + static_cast<int>(sizeof(EpiShared)) +
                                            (2 * C::kStages + 6) * 8 + 32);
  auto kern = indexer_topk_kernel<H, D, MX>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("indexer smem attribute: ") + cudaGetErrorString(e));
  e = launch_pdl(kern, dim3(grid), dim3(kThreads), smem, stream, tq, tk, p);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("indexer launch: ") + cudaGetErrorString(e));
  return DSA_OK;
}

}  // namespace

bool indexer_supported(int H, int d, int k) {
  const bool h_ok = H == 4 || H == 8 || H == 16 || H == 32 || H == 64;
  const bool d_ok = d == 32 || d == 64 || d == 128;
  return h_ok && d_ok && k >= 1 && k <= kMaxK;
}

IndexerPlan indexer_plan(int B, int Lq, int Lk, int start_pos, int k, long long rows_in) {
  (void)Lk;
  IndexerPlan pl{};
  pl.n_qblocks = (Lq + kQB - 1) / kQB;
  const int t_max = start_pos + Lq - 1;
  const int max_tiles = t_max > 0 ? (t_max + kTileK - 1) / kTileK : 0;
  const long long base_items = static_cast<long long>(B) * pl.n_qblocks;
  int S = 1;
  if (base_items < 148) {
    S = static_cast<int>(148 / base_items);
    S = std::min(S, std::max(1, max_tiles / 8));
    S = std::min(S, kMaxSplits);
  }
  pl.S = S;
  const int tiles_per_split = max_tiles > 0 ? (max_tiles + S - 1) / S : 1;
  pl.split_len = tiles_per_split * kTileK;
  pl.n_items = static_cast<int>(base_items * S);
  pl.grid = std::min(pl.n_items, kMaxGrid);
  pl.cap = cap_for(k);
  pl.cand_bytes = static_cast<size_t>(kMaxGrid) * kQB * pl.cap * 8;
  const size_t rows = rows_in >= 0 ? static_cast<size_t>(rows_in) : static_cast<size_t>(B) * Lq;
  pl.split_bytes = S > 1 ? rows * S * k * 8 : 0;
  pl.split_cnt_bytes = S > 1 ? ((rows * S * 4 + 255) / 256) * 256 : 0;
  pl.total_bytes = pl.cand_bytes + pl.split_bytes + pl.split_cnt_bytes;
  return pl;
}

// Decode rows of a varlen batch: one query row per sequence (max_Lq = 1 and
// total_q = B) against caches the decode kernels can slice.
static bool varlen_decode_applies(int B, int max_Lq, int max_Lk, int total_q, int H, int d) {
  return max_Lq == 1 && total_q == B && decode_indexer_applies(1, max_Lk, max_Lk, H, d);
}

size_t indexer_varlen_ws_bytes(int B, int max_Lq, int max_Lk, int total_q, int H, int d, int k) {
  if (varlen_decode_applies(B, max_Lq, max_Lk, total_q, H, d)) return decode_indexer_ws_bytes(B, max_Lk);
  // every row sees at most max_Lk positions
  return indexer_plan(B, max_Lq, max_Lk, std::max(0, max_Lk - max_Lq + 1), std::min(k, kMaxK), total_q)
      .total_bytes;
}

dsa_status indexer_topk_launch(const dsa_bf16* q_idx, const dsa_bf16* k_idx, const float* w,
                               int B, int Lq, int Lk, int start_pos, int H, int d, int k,
                               int32_t* idx, void* ws, size_t ws_bytes, cudaStream_t stream,
                               const VarlenArgs* vl) {
  if (vl) {
    if (varlen_decode_applies(B, Lq, Lk, vl->total_q, H, d) && ws_bytes >= decode_indexer_ws_bytes(B, Lk)) {
      const DecodeVarlen dv{vl->sp, vl->cu_k, vl->total_k};
      return decode_indexer_launch(q_idx, k_idx, w, B, Lk, 0, H, d, k, idx, ws, ws_bytes, stream, &dv);
    }
    // the plan covers rows up to t = Lk (no row sees more than its cache)
    start_pos = std::max(0, Lk - Lq + 1);
  } else if (decode_indexer_applies(Lq, Lk, start_pos, H, d) && ws_bytes >= decode_indexer_ws_bytes(B, Lk)) {
    return decode_indexer_launch(q_idx, k_idx, w, B, Lk, start_pos, H, d, k, idx, ws, ws_bytes, stream);
  }
  const long long rows = vl ? static_cast<long long>(vl->total_q) : static_cast<long long>(B) * Lq;
  IndexerPlan pl = indexer_plan(B, Lq, Lk, start_pos, k, rows);
  if (ws_bytes < pl.total_bytes) return set_error(DSA_ERR_WORKSPACE, "indexer workspace too small");
  const int sms = device_sm_count();
  if (sms <= 0) return set_error(DSA_ERR_CUDA, "cannot query the device SM count");
  const int grid = std::max(1, std::min(pl.grid, sms));

  const int chunk = d < 64 ? d : 64;
  const CUtensorMapSwizzle swz = chunk == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUtensorMap tq, tk;
  // uniform: [B][Lq * H][d] and [B][Lk][d]; varlen: one batch of the packed rows
  const uint64_t qrows = vl ? static_cast<uint64_t>(vl->total_q) * H : static_cast<uint64_t>(Lq) * H;
  const uint64_t krows = vl ? static_cast<uint64_t>(vl->total_k) : static_cast<uint64_t>(Lk);
  const uint64_t nb = vl ? 1u : static_cast<uint64_t>(B);
  if (!encode_tiled_3d(&tq, q_idx, d, qrows, nb, static_cast<uint64_t>(d) * 2, qrows * d * 2, chunk, 4 * H, swz))
    return set_error(DSA_ERR_CUDA, "tensor map for q_idx failed");
  if (!encode_tiled_3d(&tk, k_idx, d, krows, nb, static_cast<uint64_t>(d) * 2, krows * d * 2, chunk, kTileK, swz))
    return set_error(DSA_ERR_CUDA, "tensor map for k_idx failed");

  Params p{};
  uint8_t* base = static_cast<uint8_t*>(ws);
  p.w = w;
  p.idx = idx;
  p.cand = reinterpret_cast<uint64_t*>(base);
  p.split_out = pl.S > 1 ? reinterpret_cast<uint64_t*>(base + pl.cand_bytes) : nullptr;
  p.split_cnt = pl.S > 1 ? reinterpret_cast<int*>(base + pl.cand_bytes + pl.split_bytes) : nullptr;
  p.err = device_error_word();
  if (!p.err) return set_error(DSA_ERR_CUDA, "cannot resolve the device error word");
  p.cu_q = vl ? vl->cu_q : nullptr;
  p.cu_k = vl ? vl->cu_k : nullptr;
  p.sp = vl ? vl->sp : nullptr;
  p.B = B; p.Lq = Lq; p.Lk = Lk; p.start_pos = start_pos; p.k = k; p.cap = pl.cap;
  p.S = pl.S; p.split_len = pl.split_len; p.n_qblocks = pl.n_qblocks; p.n_items = pl.n_items;

  dsa_status st = DSA_ERR_UNSUPPORTED;
#define DSA_CASE(HH, DD) \
  if (H == HH && d == DD) st = launch_hd<HH, DD, false>(tq, tk, p, grid, stream);
  DSA_CASE(4, 32) DSA_CASE(4, 64) DSA_CASE(4, 128)
  DSA_CASE(8, 32) DSA_CASE(8, 64) DSA_CASE(8, 128)
  DSA_CASE(16, 32) DSA_CASE(16, 64) DSA_CASE(16, 128)
  DSA_CASE(32, 32) DSA_CASE(32, 64) DSA_CASE(32, 128)
  DSA_CASE(64, 32) DSA_CASE(64, 64) DSA_CASE(64, 128)
#undef DSA_CASE
  if (st != DSA_OK) return st == DSA_ERR_UNSUPPORTED ? set_error(st, "indexer shape unsupported") : st;
  if (pl.S > 1) {
    const int msmem = pl.S * k * 4;
    if (msmem > 48 * 1024) {
      cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(indexer_merge_kernel), msmem);
      if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("merge smem attribute: ") + cudaGetErrorString(e));
    }
    cudaError_t e = launch_pdl(indexer_merge_kernel, dim3(static_cast<unsigned>(rows)),
                               dim3(kMergeThreads), msmem, stream, p.split_out, p.split_cnt, idx, pl.S, k);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("merge launch: ") + cudaGetErrorString(e));
  }
  return DSA_OK;
}

// The low-precision selector ("注意力机制中的 Index" §5.4): the same fused
// indexer + top-k over MX operands (H_I = 64, d_I = 128, uniform batches).
// codes_q [B][Lq * 64][128] and codes_k [B][Lk][128] hold one element code
// per byte; sfq [B][sfq_groups] and sfk [B][sfk_tiles] hold the block scales
// of each group of 128 rows in the layout the TMEM copy reads (row 32c + l of
// the group, block n at byte 16 l + 4 c + n).  The workspace starts with the
// plan's candidate and split buffers.
dsa_status indexer_topk_mx_launch(const uint8_t* codes_q, const uint8_t* codes_k, const uint8_t* sfq,
                                  const uint8_t* sfk, int sfq_groups, int sfk_tiles, const float* w, int B, int Lq,
                                  int Lk, int start_pos, int fmt_code, int k, int32_t* idx, void* ws,
                                  size_t ws_bytes, cudaStream_t stream) {
  constexpr int H = 64, d = 128;
  const long long rows = static_cast<long long>(B) * Lq;
  IndexerPlan pl = indexer_plan(B, Lq, Lk, start_pos, k, rows);
  if (ws_bytes < pl.total_bytes) return set_error(DSA_ERR_WORKSPACE, "low-precision indexer workspace too small");
  const int sms = device_sm_count();
  if (sms <= 0) return set_error(DSA_ERR_CUDA, "cannot query the device SM count");
  const int grid = std::max(1, std::min(pl.grid, sms));
  CUtensorMap tq, tk;
  const uint64_t qrows = static_cast<uint64_t>(Lq) * H;
  if (!encode_tiled_3d(&tq, codes_q, d, qrows, B, d, qrows * d, d, Cfg<H, d, true>::kUnitRows,
                       CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_DATA_TYPE_UINT8))
    return set_error(DSA_ERR_CUDA, "tensor map for the query codes failed");
  if (!encode_tiled_3d(&tk, codes_k, d, Lk, B, d, static_cast<uint64_t>(Lk) * d, d, kTileK,
                       CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_DATA_TYPE_UINT8))
    return set_error(DSA_ERR_CUDA, "tensor map for the key codes failed");
  Params p{};
  uint8_t* base = static_cast<uint8_t*>(ws);
  p.w = w;
  p.idx = idx;
  p.cand = reinterpret_cast<uint64_t*>(base);
  p.split_out = pl.S > 1 ? reinterpret_cast<uint64_t*>(base + pl.cand_bytes) : nullptr;
  p.split_cnt = pl.S > 1 ? reinterpret_cast<int*>(base + pl.cand_bytes + pl.split_bytes) : nullptr;
  p.err = device_error_word();
  if (!p.err) return set_error(DSA_ERR_CUDA, "cannot resolve the device error word");
  p.B = B; p.Lq = Lq; p.Lk = Lk; p.start_pos = start_pos; p.k = k; p.cap = pl.cap;
  p.S = pl.S; p.split_len = pl.split_len; p.n_qblocks = pl.n_qblocks; p.n_items = pl.n_items;
  p.sfq = sfq; p.sfk = sfk; p.sfq_groups = sfq_groups; p.sfk_tiles = sfk_tiles;
  p.mx_idesc = make_idesc_mx(128, fmt_code, fmt_code);
  dsa_status st = launch_hd<H, d, true>(tq, tk, p, grid, stream);
  if (st != DSA_OK) return st;
  if (pl.S > 1) {
    const int msmem = pl.S * k * 4;
    if (msmem > 48 * 1024) {
      cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(indexer_merge_kernel), msmem);
      if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("merge smem attribute: ") + cudaGetErrorString(e));
    }
    cudaError_t e = launch_pdl(indexer_merge_kernel, dim3(static_cast<unsigned>(rows)), dim3(kMergeThreads), msmem,
                               stream, p.split_out, p.split_cnt, idx, pl.S, k);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("merge launch: ") + cudaGetErrorString(e));
  }
  return DSA_OK;
}

}  // namespace dsa
