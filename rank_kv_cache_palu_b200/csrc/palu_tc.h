// Host-side interface of the tcgen05/TMA (sm_100a) kernels.
#pragma once

#include <cuda_runtime.h>

#include "palu_internal.h"

namespace palu {

// Decode: shapes the tensor-core split kernel takes.
bool tc_decode_supported(const palu_config* c);
// Head blocks per group the split kernel's grid uses (heads per CTA = 2).
int tc_head_blocks(const palu_config* c);
cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t st);
// The int4-latent instantiations (own translation unit); launch_decode_tc calls it.
cudaError_t launch_decode_tc_int4(const DecodeArgs& a, cudaStream_t st);

// Decode without RoPE: the key up-projection folded into the query, scores
// taken on the cached latents (no key is rebuilt).  Its workspace adds the
// folded queries after the split partials.
bool fused_decode_supported(const palu_config* c);
size_t fused_query_bytes(const palu_config* c, int batch);
// Queries of one sequence the fused kernel serves in one pass over the cache
// (a pass takes 1, 2 or this many; DecodeArgs::qn).
int fused_queries_per_pass();
cudaError_t launch_decode_fused(const DecodeArgs& a, cudaStream_t st);

// Compress: shapes the tensor-core GEMM takes, and the scratch it needs.
bool tc_compress_supported(const palu_config* c, int n_tokens, int d_model);
// ncols_k / ncols_v: output columns of the launch (Σ of its groups' key / value ranks)
size_t tc_compress_scratch_bytes(const palu_config* c, int n_tokens, int d_model, int ncols_k, int ncols_v);
cudaError_t launch_compress_tc(const CompressArgs& a, cudaStream_t st);

}  // namespace palu
