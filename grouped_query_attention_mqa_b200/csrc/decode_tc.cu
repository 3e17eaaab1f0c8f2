// Tensor-core (tcgen05) split-KV decode: not built yet.
#include "common.cuh"

namespace mqa {

bool tc_supported(int, int) { return false; }
int tc_ctas_per_sm(int) { return 1; }
cudaError_t launch_decode_tc(const DecodeArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace mqa
