// dsa_internal.h -- host-side helpers shared by the library's translation
// units (not part of the public C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

#include "../../include/dsa.h"

namespace dsa {

// Records a message for dsa_last_error() and returns `st`.
dsa_status set_error(dsa_status st, const std::string& msg);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda
// link dependency).  Returns false on failure.
bool encode_tiled_2d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1,
                     uint64_t stride1_bytes, uint32_t box0, uint32_t box1,
                     CUtensorMapSwizzle swizzle);
bool encode_tiled_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                     uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0, uint32_t box1,
                     CUtensorMapSwizzle swizzle,
                     CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);

// Raises a kernel's dynamic shared-memory limit to at least `bytes` on the
// current device, calling the runtime only the first time per (device, kernel)
// and size (launch paths stay cheap when called every layer).
cudaError_t ensure_smem_limit(const void* func, int bytes);

// SM count of the current device (cached per device).
int device_sm_count();

// Device address of the library's error word on the current device.
unsigned int* device_error_word();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Launches a kernel as a programmatic dependent of the previous work in the
// stream: it may be scheduled before that work completes and must execute
// pdl_wait() before reading anything that work produced.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// A variable-length batch of packed rows (the public dsa_varlen, checked):
// sequence b's query rows are cu_q[b] .. cu_q[b+1]-1, its cached rows
// cu_k[b] .. cu_k[b+1]-1, its first query row at position sp[b].  The launch
// functions take the batch's maxima as Lq and Lk and a null pointer for a
// uniform batch.
struct VarlenArgs {
  const int* cu_q;
  const int* cu_k;
  const int* sp;
  int total_q, total_k;
};

// ---- indexer + top-k (indexer_topk.cu)
struct IndexerPlan {
  int S;           // key splits per query block
  int split_len;   // keys per split (multiple of 128)
  int n_qblocks;   // query blocks of 8 rows per sequence
  int n_items;     // B * n_qblocks * S
  int grid;        // persistent CTAs
  int cap;         // candidate-buffer capacity per query slot (entries)
  size_t cand_bytes, split_bytes, split_cnt_bytes, total_bytes;
};
bool indexer_supported(int H, int d, int k);
// rows: the query rows of the whole batch (B * Lq, or the packed total)
IndexerPlan indexer_plan(int B, int Lq, int Lk, int start_pos, int k, long long rows = -1);
size_t indexer_varlen_ws_bytes(int B, int max_Lq, int max_Lk, int total_q, int H, int d, int k);
dsa_status indexer_topk_launch(const dsa_bf16* q_idx, const dsa_bf16* k_idx, const float* w,
                               int B, int Lq, int Lk, int start_pos, int H, int d, int k,
                               int32_t* idx, void* ws, size_t ws_bytes, cudaStream_t stream,
                               const VarlenArgs* vl = nullptr);

// ---- low-precision selector (indexer_topk.cu kernel over MX operands,
// lowprec.cu quantisation and entry points)
dsa_status indexer_topk_mx_launch(const uint8_t* codes_q, const uint8_t* codes_k, const uint8_t* sfq,
                                  const uint8_t* sfk, int sfq_groups, int sfk_tiles, const float* w, int B, int Lq,
                                  int Lk, int start_pos, int fmt_code, int k, int32_t* idx, void* ws,
                                  size_t ws_bytes, cudaStream_t stream);

// ---- decode indexer + top-k (decode_indexer.cu): one query row per sequence
// against a long cache; used by indexer_topk_launch when it applies and the
// workspace holds a row of score keys per sequence.
bool decode_indexer_applies(int Lq, int Lk, int start_pos, int H, int d);
size_t decode_indexer_ws_bytes(int B, int Lk);
// Decode rows of a variable-length batch: row b (one per sequence) sits at
// t = sp[b] and sees the packed keys cu_k[b] .. cu_k[b] + t - 1.
struct DecodeVarlen {
  const int* sp;
  const int* cu_k;
  int total_k;
};
dsa_status decode_indexer_launch(const dsa_bf16* q_idx, const dsa_bf16* k_idx, const float* w, int B,
                                 int Lk, int start_pos, int H, int d, int k, int32_t* idx, void* ws,
                                 size_t ws_bytes, cudaStream_t stream, const DecodeVarlen* vl = nullptr);

// ---- sparse attention (sparse_attn.cu)
// rows: the query rows of the whole batch (B * Lq, or the packed total)
size_t sparse_attn_ws_rows(long long rows, int n_h, int D_v, int k);
size_t sparse_attn_ws_bytes(int B, int Lq, int n_h, int D_v, int k);
dsa_status sparse_attn_launch(const dsa_bf16* q, const dsa_bf16* kbuf, int64_t k_row_stride,
                              const dsa_bf16* vbuf, int64_t v_row_stride, const int32_t* idx,
                              int B, int Lq, int Lk, int start_pos, int n_h, int D_qk, int D_v,
                              int k, float scale, dsa_bf16* out, float* lse, void* ws,
                              size_t ws_bytes, cudaStream_t stream, const VarlenArgs* vl = nullptr);

}  // namespace dsa
