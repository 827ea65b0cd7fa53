// Tensor-core split kernel of the decode step, 16-bit latents (fp16 / bf16),
// and the shape check and dispatch for every latent kind.  The kernel itself
// is in decode_tc_kernel.cuh; int4 latents are instantiated in decode_tc_int4.cu.
//
// Method: "PALU 论文低秩投影分解" §低秩投影分解 and §把它放进一次真实推理流程里看,
// Decode 阶段 (keys rebuilt from the cached latents tile by tile, values kept in
// latent space).
#include "decode_tc_kernel.cuh"

namespace palu {

bool tc_decode_supported(const palu_config* c) {
  if (c->head_dim != 128 || c->page_size != kTile) return false;
  if (c->group_size % 2 != 0) return false;
  if (c->act_dtype != PALU_F16 && c->act_dtype != PALU_BF16) return false;
  if (c->latent_dtype == PALU_INT4) {
    // one 128-byte row of codes per token and side: rank 256 for keys and values
    if (c->rank_k != 256 || c->rank_v != 256) return false;
  } else {
    if (c->latent_dtype != c->act_dtype) return false;
    if (c->rank_k % 64 != 0 || c->rank_k > 256) return false;
    if (c->rank_v != 128 && c->rank_v != 256) return false;
  }
  const Smem L = smem_layout(c->rank_k, c->latent_dtype == PALU_INT4);
  return L.total + 1024 <= 227 * 1024;
}

int tc_head_blocks(const palu_config* c) { return c->group_size / 2; }

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t st) {
  if (a.gs % 2 != 0) return cudaErrorInvalidValue;
  if (a.lat == PALU_INT4) return launch_decode_tc_int4(a, st);
  if (a.act == PALU_BF16)
    return a.r_v == 256 ? launch_t<PALU_BF16, 2, PALU_BF16>(a, st) : launch_t<PALU_BF16, 1, PALU_BF16>(a, st);
  return a.r_v == 256 ? launch_t<PALU_F16, 2, PALU_F16>(a, st) : launch_t<PALU_F16, 1, PALU_F16>(a, st);
}

}  // namespace palu
