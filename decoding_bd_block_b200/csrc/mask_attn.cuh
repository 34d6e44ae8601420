// The 2L x 2L complementary-mask attention with views that share a sample
// (mask_attn_tc.cu, attn_simt.cu): `views` consecutive entries of the batch
// are views of one training sample whose clean halves (rows L..2L-1 of q, k
// and v) are equal, so the clean rows of the output are equal too.
#pragma once

#include "bd_common.cuh"

namespace bd {

// Tensor-core kernel: the clean query tiles of a sample are computed once
// (on its first view) and stored into every view's rows.  views must divide
// n_seqs.
cudaError_t launch_mask_attn_tc_views(const bd_attn_shape& sh, const void* q, const void* k,
                                      const void* v, void* out, int n_seqs, int views, int L,
                                      int block, int32_t* status, cudaStream_t st);

// Dispatch: the tensor-core kernel where it applies; the CUDA-core kernel
// otherwise, which computes every view's rows from its own inputs.
cudaError_t launch_block_mask_attn_views(const bd_attn_shape& sh, const void* q, const void* k,
                                         const void* v, void* out, int n_seqs, int views, int L,
                                         int block, cudaStream_t st);

}  // namespace bd
