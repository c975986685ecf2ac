// sm100.cuh -- tensor-core (tcgen05) kernels for the DeepSeek-V3 head shapes.
#pragma once

#include "common.cuh"
#include "mla.h"

namespace mla {
namespace sm100 {

inline bool supports(int H, int C, int Dn, int R, int Dv) { return false; }
inline int prefill_splits() { return 1; }
inline int auto_decode_splits(int batch, int64_t max_seqlen_k, int sms) { return 1; }
inline size_t workspace_bytes(int H, int C, int batch, int64_t n_q_rows, int64_t max_seqlen_k, int splits,
                              bool decode) { return 0; }
inline mla_status_t absorb_q(const void*, int64_t, const void*, void*, int64_t, int, cudaStream_t) {
  return MLA_ERR_UNSUPPORTED;
}
inline mla_status_t out_proj(const void*, const void*, void*, int64_t, int, cudaStream_t) { return MLA_ERR_UNSUPPORTED; }
inline mla_status_t attention(const void*, const void*, int64_t, const void*, const void*, const int32_t*,
                              const int32_t*, int, int64_t, int64_t, int64_t, int, float, void*, void*, cudaStream_t) {
  return MLA_ERR_UNSUPPORTED;
}

}  // namespace sm100
}  // namespace mla
