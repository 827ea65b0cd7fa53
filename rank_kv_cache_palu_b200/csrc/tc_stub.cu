// Placeholder for the tensor-core kernels while they are being written.
#include "palu_tc.h"

namespace palu {
bool tc_decode_supported(const palu_config*) { return false; }
int tc_head_blocks(const palu_config*) { return 2; }
cudaError_t launch_decode_tc(const DecodeArgs&, cudaStream_t) { return cudaErrorNotSupported; }
bool tc_compress_supported(const palu_config*, int, int) { return false; }
size_t tc_compress_scratch_bytes(const palu_config*, int, int) { return 0; }
cudaError_t launch_compress_tc(const CompressArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace palu
