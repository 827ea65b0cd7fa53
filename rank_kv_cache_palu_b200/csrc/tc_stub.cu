// Compress on tensor cores is not built yet: every compress call takes the
// CUDA-core kernel.
#include "palu_tc.h"

namespace palu {
bool tc_compress_supported(const palu_config*, int, int) { return false; }
size_t tc_compress_scratch_bytes(const palu_config*, int, int) { return 0; }
cudaError_t launch_compress_tc(const CompressArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace palu
