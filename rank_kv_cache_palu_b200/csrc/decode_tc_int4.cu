// Tensor-core split kernel of the decode step, int4 latents (r_k = r_v = 256):
// the instantiations of decode_tc_kernel.cuh whose warps convert the codes
// (code × fp16 scale, rounded to the compute dtype) into the MMA operand rings.
//
// Method: "PALU 论文低秩投影分解" §低秩投影分解 and §把它放进一次真实推理流程里看,
// Decode 阶段; the pages' note that the low-rank cache stacks with KV quantisation.
#include "decode_tc_kernel.cuh"

namespace palu {

cudaError_t launch_decode_tc_int4(const DecodeArgs& a, cudaStream_t st) {
  if (a.gs % 2 != 0 || a.r_k != 256 || a.r_v != 256) return cudaErrorInvalidValue;
  return a.act == PALU_BF16 ? launch_t<PALU_BF16, 2, PALU_INT4>(a, st) : launch_t<PALU_F16, 2, PALU_INT4>(a, st);
}

}  // namespace palu
