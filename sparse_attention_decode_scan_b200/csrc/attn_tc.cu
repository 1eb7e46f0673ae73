// placeholder: tensor-core sparse attention
#include "internal.h"
namespace lsa {
bool attn_tc_shape_ok(int32_t, int32_t, int32_t, int32_t, int32_t) { return false; }
int attn_tc_launches(int32_t, int32_t, int32_t) { return 2; }
bool attn_tc_supported(const AttnArgs&) { return false; }
size_t attn_tc_ws_bytes(int32_t, int32_t, int32_t, int32_t, int32_t) { return 0; }
cudaError_t launch_attn_tc(const AttnArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace lsa
