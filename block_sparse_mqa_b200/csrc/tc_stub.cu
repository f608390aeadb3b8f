// Placeholder tensor-core entry points (replaced by the tcgen05 kernels).
#include "hs_internal.h"
namespace hs {
bool tc_block_score_supported(int, int, int, int) { return false; }
size_t tc_block_score_workspace(int, int, int, int) { return 0; }
cudaError_t launch_tc_block_score(const ScoreArgs&, long long, cudaStream_t) { return cudaErrorNotSupported; }
bool tc_attention_supported(int, int, int, int, bool) { return false; }
cudaError_t launch_tc_attention(const AttnArgs&, bool, long long, cudaStream_t) { return cudaErrorNotSupported; }
}
