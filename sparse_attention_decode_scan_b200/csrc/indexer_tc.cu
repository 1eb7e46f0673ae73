// placeholder: tensor-core indexer
#include "internal.h"
namespace lsa {
bool scores_tc_shape_ok(int32_t, int32_t, int32_t, int32_t, int32_t) { return false; }
int scores_tc_launches(bool) { return 1; }
bool scores_tc_supported(const ScoresArgs&) { return false; }
size_t scores_tc_ws_bytes(int32_t, bool) { return 0; }
cudaError_t launch_scores_tc(const ScoresArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace lsa
