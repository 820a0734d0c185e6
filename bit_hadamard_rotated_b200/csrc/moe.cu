// moe.cu -- hq_moe_experts (placeholder until the expert-grouped kernels land).
#include "hq_internal.h"

extern "C" {

size_t hq_moe_workspace_size(int n_experts, int hidden, int inter, int T, int k) {
  (void)n_experts;
  (void)hidden;
  (void)inter;
  (void)T;
  (void)k;
  return 0;
}

hq_status hq_moe_experts(const hq_expert* experts, int n_experts, int hidden, int inter,
                         const uint16_t* x, int T, const int32_t* topk_ids, const float* topk_w,
                         int k, const int8_t* signs_in, const int8_t* signs_mid, float* y,
                         void* workspace, size_t ws_bytes, hq_stream_t stream) {
  (void)experts; (void)n_experts; (void)hidden; (void)inter; (void)x; (void)T; (void)topk_ids;
  (void)topk_w; (void)k; (void)signs_in; (void)signs_mid; (void)y; (void)workspace;
  (void)ws_bytes; (void)stream;
  return HQ_ERR_UNSUPPORTED;
}

}  // extern "C"
