// sparse_attn.cu -- sparse MLA core attention (placeholder until the kernel lands).
#include "dsa_internal.h"

namespace dsa {

size_t sparse_attn_ws_bytes(int, int, int, int, int) { return 0; }

dsa_status sparse_attn_launch(const dsa_bf16*, const dsa_bf16*, int64_t, const dsa_bf16*, int64_t,
                              const int32_t*, int, int, int, int, int, int, int, int, float,
                              dsa_bf16*, float*, void*, size_t, cudaStream_t) {
  return set_error(DSA_ERR_UNSUPPORTED, "dsa_sparse_attn: not built yet");
}

}  // namespace dsa
